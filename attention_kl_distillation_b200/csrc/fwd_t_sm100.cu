// fwd_t_sm100.cu -- attention-KL forward for few query rows, keys on the UMMA
// M axis, for sm_100a.
//
// Same result as fwd_sm100.cu (StreamKL summary page, "Metodologia" section 1:
// five running scalars per query row, L = acc/l1 + LSE2 - LSE1).  The tile is
// transposed as in the ETAP page's core mechanism (S^T = K Q^T, so the long key
// axis is the MMA's M dimension and the short query axis its N): with a
// 128-row query tile and N_Q <= 32, most of the rows would be padding and all
// real rows would sit in one SM sub-partition's TMEM lanes.
//
// B200 mapping (one CTA per SM, persistent):
//   work unit   (bh, query group of NQT = 16 or 32 rows, key chunk)
//   warp 0      TMA producer: the group's Q1/Q2 rows once per unit, then the
//               K1/K2 tiles (128 keys) of the chunk into a ring whose K1 and K2
//               halves fill and free separately (128-byte swizzle, no multicast)
//   warp 1      TMEM owner and UMMA issuer: per key tile S1^T = K1 Q1^T and
//               S2^T = K2 Q2^T (M = 128 keys, N = NQT, both operands in shared
//               memory, fp32 accumulators) into one of NSLOT TMEM slots
//   warps 2..17 four reduction warpgroups; thread k owns key lane k of every
//               key tile, warpgroup g owns queries [g*QT, (g+1)*QT) of the
//               group.  Each thread keeps, per query, the running state of the
//               keys it has seen (one element per key tile); at the end of the
//               unit the 128 key lanes merge their states (shuffles within a
//               warp, shared memory across the four warps) with the same
//               rescaling as the split-K merge.
// One exponential per element and distribution: with d = x - m, the new
// element and the old state's rescale factor are 2^min(d,0) and 2^min(-d,0),
// one of which is 1.
// TMEM: slot s holds S1^T in [s*2*NQT, s*2*NQT + NQT) and S2^T after it.
#include "kernels.h"
#include "sm100.cuh"

#include <cmath>

namespace skl {
namespace {

constexpr int BK = kFwdBK;      // keys per tile (UMMA M)
constexpr int NRW = 4;          // reduction warpgroups
constexpr int NSLOT = 4;        // TMEM slots of S tiles
constexpr int NTHREADS = 64 + NRW * 128;
constexpr float kLn2 = 0.6931471805599453f;

template <int D1, int D2, int NQT>
struct FwdTLayout {
  static constexpr int k1_bytes = BK * D1 * 2;
  static constexpr int k2_bytes = BK * D2 * 2;
  static constexpr int stage_bytes = k1_bytes + k2_bytes;
  static constexpr int q1_bytes = NQT * D1 * 2;
  static constexpr int q2_bytes = NQT * D2 * 2;
  static constexpr int QT = NQT / NRW;  // queries per reduction thread
  static constexpr int merge_bytes = NRW * 4 * QT * 5 * 4;  // [wg][quarter][query][5] fp32
  static constexpr int fixed = q1_bytes + q2_bytes + merge_bytes + 1024 + 512;
  static constexpr int ks_fit = (232448 - fixed) / stage_bytes;
  static constexpr int KSTAGES = ks_fit > 6 ? 6 : ks_fit;
  static constexpr int k_off = 0;
  static constexpr int q_off = k_off + KSTAGES * stage_bytes;
  static constexpr int merge_off = q_off + q1_bytes + q2_bytes;
  static constexpr int bar_off = merge_off + merge_bytes;
  // barriers: qfull, qempty, kfull[KS][2], kempty[KS][2], sfull[NSLOT], sempty[NSLOT], drain
  static constexpr int nbar = 3 + 4 * KSTAGES + 2 * NSLOT;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int total = misc_off + 16;
  static constexpr int alloc = total + 1024;
  static constexpr uint32_t tmem_cols = NSLOT * 2 * NQT;  // 128 or 256
  static_assert(KSTAGES >= 3, "key ring too shallow");
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(q1_bytes % 1024 == 0 && k1_bytes % 1024 == 0 && k2_bytes % 1024 == 0 &&
                    (q_off % 1024) == 0,
                "operand tiles must keep 1024-byte alignment for the 128B swizzle atoms");
  static_assert(tmem_cols == 128 || tmem_cols == 256, "TMEM allocation is a power of two");
};

// Work unit u: split c fastest, then query group g, then head bh.
struct UnitT {
  int bh, g, kt_lo, kt_end;  // key tiles [kt_lo, kt_end) are visible to some row of the group
  int split;
};

__device__ __forceinline__ UnitT decode_unit_t(const FwdParams& p, int nqt, int u) {
  const int ngroups = (p.NQ + nqt - 1) / nqt;
  const int ns = p.nsplit > 1 ? p.nsplit : 1;
  UnitT w;
  w.split = u % ns;
  u /= ns;
  w.g = u % ngroups;
  w.bh = u / ngroups;
  const int nkt_all = (p.NK + BK - 1) / BK;
  w.kt_lo = p.nsplit > 1 ? w.split * p.kt_chunk : 0;
  const int kt_hi = p.nsplit > 1 ? min(nkt_all, w.kt_lo + p.kt_chunk) : nkt_all;
  w.kt_end = kt_hi;
  if (p.causal) {
    const int last_row = min(p.NQ - 1, (w.g + 1) * nqt - 1);
    w.kt_end = min(kt_hi, (last_row + p.NK - p.NQ) / BK + 1);
  }
  return w;
}

struct QState {
  float m1, m2, l1, l2, acc;
};

// Adds one element (base-2 logits x1, x2) to a running state.  With
// d = x - m, exactly one of the new weight and the old state's factor is 1 and
// the other is 2^-|d|; a state that has seen nothing (m = -inf) gets factor 0.
__device__ __forceinline__ void add_element(QState& s, float x1, float x2) {
  const float d1 = x1 - s.m1, d2 = x2 - s.m2;
  const float e1 = ex2(-fabsf(d1)), e2 = ex2(-fabsf(d2));
  const bool up1 = d1 > 0.f, up2 = d2 > 0.f;
  const float a1 = up1 ? e1 : 1.f, p1 = up1 ? 1.f : e1;
  const float a2 = up2 ? e2 : 1.f, p2 = up2 ? 1.f : e2;
  s.acc = fmaf(s.acc, a1, p1 * (x1 - x2));
  s.l1 = fmaf(s.l1, a1, p1);
  s.l2 = fmaf(s.l2, a2, p2);
  s.m1 = up1 ? x1 : s.m1;
  s.m2 = up2 ? x2 : s.m2;
}

// Merges state o into s (the split-K merge rule).
__device__ __forceinline__ void merge_state(QState& s, const QState& o) {
  const float m1 = fmaxf(s.m1, o.m1), m2 = fmaxf(s.m2, o.m2);
  const float fa1 = s.m1 == -INFINITY ? 0.f : ex2(s.m1 - m1);
  const float fb1 = o.m1 == -INFINITY ? 0.f : ex2(o.m1 - m1);
  const float fa2 = s.m2 == -INFINITY ? 0.f : ex2(s.m2 - m2);
  const float fb2 = o.m2 == -INFINITY ? 0.f : ex2(o.m2 - m2);
  s.l1 = fmaf(s.l1, fa1, o.l1 * fb1);
  s.l2 = fmaf(s.l2, fa2, o.l2 * fb2);
  s.acc = fmaf(s.acc, fa1, o.acc * fb1);
  s.m1 = m1;
  s.m2 = m2;
}

template <int D1, int D2, int NQT>
__global__ void __launch_bounds__(NTHREADS, 1) streamkl_fwd_t_kernel(const __grid_constant__ FwdParams p) {
  using Lay = FwdTLayout<D1, D2, NQT>;
  constexpr int KS = Lay::KSTAGES;
  constexpr int QT = Lay::QT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* qfull = bars + 0;
  uint64_t* qempty = qfull + 1;
  uint64_t* kfull = qempty + 1;        // [KS][2]
  uint64_t* kempty = kfull + 2 * KS;   // [KS][2]
  uint64_t* sfull = kempty + 2 * KS;   // [NSLOT]
  uint64_t* sempty = sfull + NSLOT;    // [NSLOT]
  uint64_t* drain = sempty + NSLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 4);
  float* merge = reinterpret_cast<float*>(smem + Lay::merge_off);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int s = 0; s < 2 * KS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4 * NRW);  // one arrival per reduction warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmK1);
    tma_prefetch_desc(&p.tmK2);
    tma_prefetch_desc(&p.tmQ1);
    tma_prefetch_desc(&p.tmQ2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int ngroups = (p.NQ + NQT - 1) / NQT;
  const int total = p.BH * ngroups * (p.nsplit > 1 ? p.nsplit : 1);
  auto k1_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes; };
  auto k2_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes + Lay::k1_bytes; };
  uint8_t* q1_s = smem + Lay::q_off;
  uint8_t* q2_s = smem + Lay::q_off + Lay::q1_bytes;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ks = 0;
      uint32_t kph = 0, qph = 0;
      uint32_t armed_k[2 * KS] = {};  // last armed phase + 1 (0 = never)
      uint32_t armed_q = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
        const UnitT w = decode_unit_t(p, NQT, u);
        if (w.kt_end <= w.kt_lo) continue;
        if (!(ok = mbar_wait(qempty, qph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(qfull, Lay::q1_bytes + Lay::q2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(q1_s + b * (NQT * 128), &p.tmQ1, qfull, b * 64, w.g * NQT, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(q2_s + b * (NQT * 128), &p.tmQ2, qfull, b * 64, w.g * NQT, w.bh);
        armed_q = qph + 1;
        qph ^= 1;
        for (int kt = w.kt_lo; kt < (p.withhold_keys ? w.kt_lo : w.kt_end); ++kt) {
          if (!(ok = mbar_wait(&kempty[2 * ks], kph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfull[2 * ks], Lay::k1_bytes);
#pragma unroll
          for (int b = 0; b < D1 / 64; ++b)
            tma_load_3d(k1_s(ks) + b * (BK * 128), &p.tmK1, &kfull[2 * ks], b * 64, kt * BK, w.bh);
          armed_k[2 * ks] = kph + 1;
          if (!(ok = mbar_wait(&kempty[2 * ks + 1], kph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfull[2 * ks + 1], Lay::k2_bytes);
#pragma unroll
          for (int b = 0; b < D2 / 64; ++b)
            tma_load_3d(k2_s(ks) + b * (BK * 128), &p.tmK2, &kfull[2 * ks + 1], b * 64, kt * BK, w.bh);
          armed_k[2 * ks + 1] = kph + 1;
          if (++ks == KS) {
            ks = 0;
            kph ^= 1;
          }
        }
      }
      if (!ok) {
        // Aborting: let the copies already in flight land before the CTA exits.
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        for (int s = 0; s < 2 * KS; ++s)
          if (armed_k[s]) mbar_wait(&kfull[s], armed_k[s] - 1, dctl);
        if (armed_q) mbar_wait(qfull, armed_q - 1, dctl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BK, NQT);  // M = 128 keys, N = NQT queries, both K-major
      const uint64_t a1 = sdesc_sw128(smem_u32(q1_s), 16, 1024);
      const uint64_t a2 = sdesc_sw128(smem_u32(q2_s), 16, 1024);
      int ks = 0, slot = 0;
      uint32_t kph = 0, qph = 0, sph = 0;  // sph: bit s = parity of slot s
      bool ok = true;
      for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
        const UnitT w = decode_unit_t(p, NQT, u);
        if (w.kt_end <= w.kt_lo) continue;
        if (!(ok = mbar_wait(qfull, qph, ctl))) break;
        qph ^= 1;
        for (int kt = w.kt_lo; kt < w.kt_end; ++kt) {
          if (!(ok = mbar_wait(&sempty[slot], ((sph >> slot) & 1u) ^ 1u, ctl))) break;
          const uint32_t d = tmem_base + slot * 2 * NQT;
          const uint64_t b1 = sdesc_sw128(smem_u32(k1_s(ks)), 16, 1024);
          const uint64_t b2 = sdesc_sw128(smem_u32(k2_s(ks)), 16, 1024);
          if (!(ok = mbar_wait(&kfull[2 * ks], kph, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D1 / 16; ++kk)
            umma_bf16_ss(d, sdesc_advance(b1, (kk >> 2) * (BK * 128) + (kk & 3) * 32),
                         sdesc_advance(a1, (kk >> 2) * (NQT * 128) + (kk & 3) * 32), idesc, kk > 0);
          umma_commit(&kempty[2 * ks]);
          if (!(ok = mbar_wait(&kfull[2 * ks + 1], kph, ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D2 / 16; ++kk)
            umma_bf16_ss(d + NQT, sdesc_advance(b2, (kk >> 2) * (BK * 128) + (kk & 3) * 32),
                         sdesc_advance(a2, (kk >> 2) * (NQT * 128) + (kk & 3) * 32), idesc, kk > 0);
          umma_commit(&kempty[2 * ks + 1]);
          umma_commit(&sfull[slot]);
          sph ^= 1u << slot;
          if (++slot == NSLOT) slot = 0;
          if (++ks == KS) {
            ks = 0;
            kph ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(qempty);  // the group's Q tiles are free once this unit's UMMAs are done
      }
      umma_commit(drain);
      volatile int zero = 0;
      WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
      mbar_wait(drain, 0, dctl);
    }
  } else {
    // ------------------------------------------------------------ reduction
    const int wg = (warp - 2) >> 2;  // queries [wg*QT, wg*QT + QT) of the group
    const int quarter = warp & 3;
    const int kl = quarter * 32 + lane;  // key lane
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int off = p.NK - p.NQ;
    float* mslot = merge + (wg * 4 + quarter) * QT * 5;  // this warp's merged states
    int slot = 0;
    uint32_t sph = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < total; u += gridDim.x) {
      const UnitT w = decode_unit_t(p, NQT, u);
      if (w.kt_end <= w.kt_lo) continue;
      const int i0 = w.g * NQT + wg * QT;  // first query row of this thread
      QState st[QT];
#pragma unroll
      for (int j = 0; j < QT; ++j) st[j] = QState{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
      for (int kt = w.kt_lo; kt < w.kt_end; ++kt) {
        if (!(ok = mbar_wait(&sfull[slot], (sph >> slot) & 1u, ctl))) break;
        tc_fence_after();
        uint32_t a[QT], b[QT];
        const uint32_t col = tlane + slot * 2 * NQT + wg * QT;
        tmem_ld_32x32b<QT>(col, a);
        tmem_ld_32x32b<QT>(col + NQT, b);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[slot]);
        sph ^= 1u << slot;
        if (++slot == NSLOT) slot = 0;
        const int key = kt * BK + kl;
        // key < NK, and with the causal mask key <= i + off for row i
        const int vis_from = p.causal ? key - off : 0;  // rows i >= vis_from see the key
        if (key < p.NK) {
#pragma unroll
          for (int j = 0; j < QT; ++j)
            if (i0 + j >= vis_from && i0 + j < p.NQ)
              add_element(st[j], __uint_as_float(a[j]) * p.c1, __uint_as_float(b[j]) * p.c2);
        }
      }
      if (!ok) break;
      // Merge the 128 key lanes: butterfly within the warp, then the four warps.
#pragma unroll
      for (int j = 0; j < QT; ++j) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          QState t;
          t.m1 = __shfl_xor_sync(0xffffffffu, st[j].m1, o);
          t.m2 = __shfl_xor_sync(0xffffffffu, st[j].m2, o);
          t.l1 = __shfl_xor_sync(0xffffffffu, st[j].l1, o);
          t.l2 = __shfl_xor_sync(0xffffffffu, st[j].l2, o);
          t.acc = __shfl_xor_sync(0xffffffffu, st[j].acc, o);
          merge_state(st[j], t);
        }
      }
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < QT; ++j) {
          mslot[j * 5 + 0] = st[j].m1;
          mslot[j * 5 + 1] = st[j].m2;
          mslot[j * 5 + 2] = st[j].l1;
          mslot[j * 5 + 3] = st[j].l2;
          mslot[j * 5 + 4] = st[j].acc;
        }
      }
      named_bar_sync(1 + wg, 128);
      if (quarter == 0 && lane < QT) {
        const int j = lane;
        const float* m0 = merge + (wg * 4) * QT * 5 + j * 5;
        QState s{m0[0], m0[1], m0[2], m0[3], m0[4]};
#pragma unroll
        for (int q = 1; q < 4; ++q) {
          const float* mq = m0 + q * QT * 5;
          merge_state(s, QState{mq[0], mq[1], mq[2], mq[3], mq[4]});
        }
        const int i = i0 + j;
        if (i < p.NQ) {
          const size_t o = static_cast<size_t>(w.bh) * p.NQ + i;
          if (p.nsplit > 1) {
            // partial state of this key chunk, merged by streamkl_fwd_merge_kernel
            const size_t rows = static_cast<size_t>(p.BH) * p.NQ;
            float* dst = p.part + static_cast<size_t>(w.split) * 5 * rows + o;
            dst[0 * rows] = s.m1;
            dst[1 * rows] = s.m2;
            dst[2 * rows] = s.l1;
            dst[3 * rows] = s.l2;
            dst[4 * rows] = s.acc;
          } else {
            const float lg1 = lg2(s.l1), lg2v = lg2(s.l2);
            p.LSE1[o] = kLn2 * (s.m1 + lg1);
            p.LSE2[o] = kLn2 * (s.m2 + lg2v);
            p.L[o] = kLn2 * (s.acc / s.l1 + (s.m2 - s.m1) + (lg2v - lg1));
          }
        }
      }
      named_bar_sync(1 + wg, 128);  // the merge slots may be reused
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Lay::tmem_cols);
  }
}

template <int D1, int D2, int NQT>
cudaError_t launch_t(const FwdParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = FwdTLayout<D1, D2, NQT>::alloc;
  auto kern = streamkl_fwd_t_kernel<D1, D2, NQT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int NQT>
cudaError_t launch_nqt(const FwdParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128, NQT>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64, NQT>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128, NQT>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64, NQT>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_fwd_t(const FwdParams& p, int d1, int d2, int nqt, int grid, cudaStream_t stream) {
  if (nqt == 16) return launch_nqt<16>(p, d1, d2, grid, stream);
  if (nqt == 32) return launch_nqt<32>(p, d1, d2, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace skl
