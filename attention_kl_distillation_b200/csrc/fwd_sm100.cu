// fwd_sm100.cu -- fused single-pass attention-KL forward for sm_100a.
//
// StreamKL summary page, "Metodologia" section 1: each query row keeps five
// running scalars (m1, m2, l1, l2, acc) while key tiles stream through on-chip
// memory, and finishes with L = acc/l1 + LSE2 - LSE1, LSE_t = m_t + log l_t.
// Key tiles past the causal frontier are never loaded or multiplied.
//
// B200 mapping (one CTA per SM, persistent):
//   warp 0      TMA producer: Q1/Q2 tile once per work unit, K1/K2 tiles into
//               a 4-stage shared-memory ring (128-byte swizzle, no multicast).
//   warp 1      TMEM owner and UMMA issuer: S1 = Q1 K1^T and S2 = Q2 K2^T for
//               each key tile (tcgen05.mma kind::f16, fp32 accumulators) into
//               one of four TMEM buffers of 2 x 64 columns.
//   warps 2..5  reduction warpgroup: thread r owns query row r (TMEM lane r),
//               loads its 64 + 64 logits with tcgen05.ld, frees the buffer and
//               applies the online update in registers (exp2 on the MUFU pipe,
//               softmax scale folded into the exponent argument).
// The accumulator acc is one fp32 per row: there is no PV product and no
// output tile, which is what lets both S tiles live in TMEM at once.
//
// Work units are (bh, 128-row query tile), visited longest first (the last
// query tiles of a causal problem see the most keys) and dealt to CTAs in a
// snake order, an approximation of longest-processing-time scheduling.
#include "kernels.h"
#include "sm100.cuh"

#include <cmath>

namespace skl {
namespace {

constexpr int BQ = kFwdBQ;
constexpr int BK = kFwdBK;
constexpr int KSTAGES = 4;            // K1/K2 shared-memory ring depth
constexpr int SBUF = 512 / (2 * BK);  // TMEM S1/S2 buffers (4 x 128 columns)
constexpr int NTHREADS = 192;
constexpr float kLn2 = 0.6931471805599453f;

template <int D1, int D2>
struct FwdLayout {
  static constexpr int q1_bytes = BQ * D1 * 2;
  static constexpr int q2_bytes = BQ * D2 * 2;
  static constexpr int k1_bytes = BK * D1 * 2;
  static constexpr int k2_bytes = BK * D2 * 2;
  static constexpr int stage_bytes = k1_bytes + k2_bytes;
  static constexpr int q1_off = 0;
  static constexpr int q2_off = q1_off + q1_bytes;
  static constexpr int k_off = q2_off + q2_bytes;
  static constexpr int bar_off = k_off + KSTAGES * stage_bytes;
  // barriers: qfull, qempty, kfull[KSTAGES], kempty[KSTAGES], sfull[SBUF], sempty[SBUF], drain
  static constexpr int nbar = 3 + 2 * KSTAGES + 2 * SBUF;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int total = misc_off + 16;
  static constexpr int alloc = total + 1024;  // slack to align the base to 1024 B
  static_assert(q1_bytes % 1024 == 0 && q2_bytes % 1024 == 0 && k1_bytes % 1024 == 0 &&
                    k2_bytes % 1024 == 0,
                "tiles must keep 1024-byte alignment for the 128B swizzle atoms");
};

struct Sched {
  int total, G, cta, round;
  __device__ bool next(int& u) {
    for (;;) {
      const int base = round * G;
      if (base >= total) return false;
      const int uu = base + ((round & 1) ? (G - 1 - cta) : cta);
      ++round;
      if (uu < total) {
        u = uu;
        return true;
      }
    }
  }
};

struct Unit {
  int bh, q0, nkt, kt_mask;  // key tiles [kt_mask, nkt) need element masks
};

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  const int nqt = (p.NQ + BQ - 1) / BQ;
  Unit w;
  w.bh = u % p.BH;
  const int qt = nqt - 1 - u / p.BH;  // longest (last) query tiles first
  w.q0 = qt * BQ;
  const int nkt_all = (p.NK + BK - 1) / BK;
  const int off = p.NK - p.NQ;
  int nkt = nkt_all;
  int kt_mask = (p.NK % BK) ? nkt_all - 1 : nkt_all;
  if (p.causal) {
    const int last = min(w.q0 + BQ - 1, p.NQ - 1) + off;  // last key any row of the tile sees
    nkt = min(nkt_all, last / BK + 1);
    kt_mask = min(kt_mask, (w.q0 + off + 1) / BK);  // first tile the first row cannot fully see
  }
  w.nkt = nkt;
  w.kt_mask = kt_mask;
  return w;
}

struct RowState {
  float m1, m2, l1, l2, acc;
};

// One key tile of the online update for one row.  a/b hold the raw fp32
// products <Q1_i, K1_j> and <Q2_i, K2_j>; c1/c2 fold the softmax scale and
// log2(e).  With MASK, only the first nv keys of the tile are visible.
template <bool MASK>
__device__ __forceinline__ void tile_update(const uint32_t (&a)[BK], const uint32_t (&b)[BK],
                                            float c1, float c2, int nv, RowState& st) {
  float mx1[4], mx2[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) mx1[k] = mx2[k] = -INFINITY;
#pragma unroll
  for (int j = 0; j < BK; ++j) {
    float v1 = __uint_as_float(a[j]), v2 = __uint_as_float(b[j]);
    if (MASK && j >= nv) v1 = v2 = -INFINITY;
    mx1[j & 3] = fmaxf(mx1[j & 3], v1);
    mx2[j & 3] = fmaxf(mx2[j & 3], v2);
  }
  const float tmx1 = fmaxf(fmaxf(mx1[0], mx1[1]), fmaxf(mx1[2], mx1[3]));
  const float tmx2 = fmaxf(fmaxf(mx2[0], mx2[1]), fmaxf(mx2[2], mx2[3]));
  const float m1n = fmaxf(st.m1, tmx1 * c1);
  const float m2n = fmaxf(st.m2, tmx2 * c2);
  // A row that has seen no key yet keeps m = -inf; shift by 0 instead so that
  // no inf - inf appears.  (Every valid row sees key 0 in its first tile.)
  const float m1u = (m1n == -INFINITY) ? 0.f : m1n;
  const float m2u = (m2n == -INFINITY) ? 0.f : m2n;
  float sp1[4], sp2[4], sd[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) sp1[k] = sp2[k] = sd[k] = 0.f;
#pragma unroll
  for (int j = 0; j < BK; ++j) {
    float t1 = fmaf(__uint_as_float(a[j]), c1, -m1u);
    float t2 = fmaf(__uint_as_float(b[j]), c2, -m2u);
    float p1 = ex2(t1), p2 = ex2(t2);
    if (MASK && j >= nv) {
      p1 = 0.f;
      p2 = 0.f;
      t1 = t2 = 0.f;
    }
    sp1[j & 3] += p1;
    sp2[j & 3] += p2;
    sd[j & 3] = fmaf(p1, t1 - t2, sd[j & 3]);
  }
  const float s1 = (sp1[0] + sp1[1]) + (sp1[2] + sp1[3]);
  const float s2 = (sp2[0] + sp2[1]) + (sp2[2] + sp2[3]);
  const float d = (sd[0] + sd[1]) + (sd[2] + sd[3]);
  const float a1 = ex2(((st.m1 == -INFINITY) ? m1u : st.m1) - m1u);
  const float a2 = ex2(((st.m2 == -INFINITY) ? m2u : st.m2) - m2u);
  // sum_j p1 (y1 - y2) with y1 - y2 = (t1 - t2) + (m1 - m2)
  st.acc = fmaf(a1, st.acc, fmaf(m1u - m2u, s1, d));
  st.l1 = fmaf(a1, st.l1, s1);
  st.l2 = fmaf(a2, st.l2, s2);
  st.m1 = m1n;
  st.m2 = m2n;
}

template <int D1, int D2>
__global__ void __launch_bounds__(NTHREADS, 1) streamkl_fwd_kernel(const __grid_constant__ FwdParams p) {
  using Lay = FwdLayout<D1, D2>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* qfull = bars + 0;
  uint64_t* qempty = bars + 1;
  uint64_t* kfull = bars + 2;
  uint64_t* kempty = kfull + KSTAGES;
  uint64_t* sfull = kempty + KSTAGES;
  uint64_t* sempty = sfull + SBUF;
  uint64_t* drain = sempty + SBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int s = 0; s < KSTAGES; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < SBUF; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4);  // one arrival per reduction warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ1);
    tma_prefetch_desc(&p.tmK1);
    tma_prefetch_desc(&p.tmQ2);
    tma_prefetch_desc(&p.tmK2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  Sched sched{fwd_units(p.BH, p.NQ), static_cast<int>(gridDim.x), static_cast<int>(blockIdx.x), 0};
  uint8_t* q1_s = smem + Lay::q1_off;
  uint8_t* q2_s = smem + Lay::q2_off;
  auto k1_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes; };
  auto k2_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes + Lay::k1_bytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ks = 0;
      uint32_t kph = 0, qph = 0;
      uint32_t armed_q = 0, armed_k[KSTAGES] = {};  // last armed phase + 1 (0 = never)
      int u;
      bool ok = true;
      while (ok && sched.next(u)) {
        const Unit w = decode_unit(p, u);
        if (!(ok = mbar_wait(qempty, qph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(qfull, Lay::q1_bytes + Lay::q2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(q1_s + b * (BQ * 128), &p.tmQ1, qfull, b * 64, w.q0, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(q2_s + b * (BQ * 128), &p.tmQ2, qfull, b * 64, w.q0, w.bh);
        armed_q = qph + 1;
        qph ^= 1;
        for (int kt = 0; kt < w.nkt; ++kt) {
          if (!(ok = mbar_wait(&kempty[ks], kph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfull[ks], Lay::stage_bytes);
#pragma unroll
          for (int b = 0; b < D1 / 64; ++b)
            tma_load_3d(k1_s(ks) + b * (BK * 128), &p.tmK1, &kfull[ks], b * 64, kt * BK, w.bh);
#pragma unroll
          for (int b = 0; b < D2 / 64; ++b)
            tma_load_3d(k2_s(ks) + b * (BK * 128), &p.tmK2, &kfull[ks], b * 64, kt * BK, w.bh);
          armed_k[ks] = kph + 1;
          if (++ks == KSTAGES) {
            ks = 0;
            kph ^= 1;
          }
        }
      }
      if (!ok) {
        // Aborting: let the copies already in flight land before the CTA exits.
        WaitCtl drainctl{abort_flag, p.status, p.wait_limit_ns};
        volatile int zero = 0;
        drainctl.abort = &zero;
        if (armed_q) mbar_wait(qfull, armed_q - 1, drainctl);
        for (int s = 0; s < KSTAGES; ++s)
          if (armed_k[s]) mbar_wait(&kfull[s], armed_k[s] - 1, drainctl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BQ, BK);
      int ks = 0, sb = 0;
      uint32_t kph = 0, sph = 0, qph = 0;
      const uint32_t q1a = smem_u32(q1_s), q2a = smem_u32(q2_s);
      int u;
      bool ok = true;
      while (ok && sched.next(u)) {
        const Unit w = decode_unit(p, u);
        if (!(ok = mbar_wait(qfull, qph, ctl))) break;
        qph ^= 1;
        tc_fence_after();
        for (int kt = 0; kt < w.nkt; ++kt) {
          if (!(ok = mbar_wait(&kfull[ks], kph, ctl))) break;
          if (!(ok = mbar_wait(&sempty[sb], sph ^ 1, ctl))) break;
          tc_fence_after();
          const uint32_t k1a = smem_u32(k1_s(ks)), k2a = smem_u32(k2_s(ks));
          const uint32_t t1 = tmem_base + sb * (2 * BK);
          const uint32_t t2 = t1 + BK;
#pragma unroll
          for (int kk = 0; kk < D1 / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            umma_bf16_ss(t1, sdesc_sw128(q1a + (kk >> 2) * (BQ * 128) + off, 16, 1024),
                         sdesc_sw128(k1a + (kk >> 2) * (BK * 128) + off, 16, 1024), idesc, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D2 / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;
            umma_bf16_ss(t2, sdesc_sw128(q2a + (kk >> 2) * (BQ * 128) + off, 16, 1024),
                         sdesc_sw128(k2a + (kk >> 2) * (BK * 128) + off, 16, 1024), idesc, kk > 0);
          }
          umma_commit(&sfull[sb]);
          umma_commit(&kempty[ks]);
          if (++ks == KSTAGES) {
            ks = 0;
            kph ^= 1;
          }
          if (++sb == SBUF) {
            sb = 0;
            sph ^= 1;
          }
        }
        if (ok) umma_commit(qempty);
      }
      // Every UMMA issued by this thread completes before TMEM is released.
      umma_commit(drain);
      WaitCtl drainctl{abort_flag, p.status, p.wait_limit_ns};
      volatile int zero = 0;
      drainctl.abort = &zero;
      mbar_wait(drain, 0, drainctl);
    }
  } else {
    // ------------------------------------------------------------ reduction
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const int off = p.NK - p.NQ;
    int sb = 0;
    uint32_t sph = 0;
    int u;
    bool ok = true;
    while (ok && sched.next(u)) {
      const Unit w = decode_unit(p, u);
      const int i_abs = w.q0 + row;
      const int lim = p.causal ? min(p.NK, i_abs + off + 1) : p.NK;  // visible keys [0, lim)
      RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
      for (int kt = 0; kt < w.nkt; ++kt) {
        if (!(ok = mbar_wait(&sfull[sb], sph, ctl))) break;
        tc_fence_after();
        uint32_t a[BK], b[BK];
        const uint32_t tcol = tlane + sb * (2 * BK);
        tmem_ld_32x32b_x32(tcol + 0, *reinterpret_cast<uint32_t(*)[32]>(&a[0]));
        tmem_ld_32x32b_x32(tcol + 32, *reinterpret_cast<uint32_t(*)[32]>(&a[32]));
        tmem_ld_32x32b_x32(tcol + BK, *reinterpret_cast<uint32_t(*)[32]>(&b[0]));
        tmem_ld_32x32b_x32(tcol + BK + 32, *reinterpret_cast<uint32_t(*)[32]>(&b[32]));
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        if (++sb == SBUF) {
          sb = 0;
          sph ^= 1;
        }
        if (kt >= w.kt_mask)
          tile_update<true>(a, b, p.c1, p.c2, lim - kt * BK, st);
        else
          tile_update<false>(a, b, p.c1, p.c2, BK, st);
      }
      if (!ok) break;
      if (i_abs < p.NQ) {
        const float lg1 = lg2(st.l1), lg2v = lg2(st.l2);
        const size_t o = static_cast<size_t>(w.bh) * p.NQ + i_abs;
        p.LSE1[o] = kLn2 * (st.m1 + lg1);
        p.LSE2[o] = kLn2 * (st.m2 + lg2v);
        p.L[o] = kLn2 * (st.acc / st.l1 + (st.m2 - st.m1) + (lg2v - lg1));
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int D1, int D2>
cudaError_t launch_t(const FwdParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = FwdLayout<D1, D2>::alloc;
  auto kern = streamkl_fwd_kernel<D1, D2>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t fwd_smem_bytes(int d1, int d2) {
  if (d1 == 128 && d2 == 128) return FwdLayout<128, 128>::alloc;
  if (d1 == 128 && d2 == 64) return FwdLayout<128, 64>::alloc;
  if (d1 == 64 && d2 == 128) return FwdLayout<64, 128>::alloc;
  if (d1 == 64 && d2 == 64) return FwdLayout<64, 64>::alloc;
  return 0;
}

cudaError_t launch_fwd(const FwdParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace skl
