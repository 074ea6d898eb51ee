// bwd_sm100.cu -- recompute backward of the fused attention-KL for sm_100a.
//
// StreamKL summary page, "Metodologia" section 2: the probabilities are
// regenerated tile by tile from the saved LSE vectors, P_t = exp(x_t - LSE_t),
// and every (query tile, key tile) pair is visited once; dQ is accumulated
// with atomics across key tiles.  With g = dL, c = L:
//
//   dS1 = g * P1 * ((x1 - LSE1) - (x2 - LSE2) - L)      (student fixed: dQ1, dK1)
//   dS2 = g * (P2 - P1)                                 (teacher fixed: dQ2, dK2)
//   dQ_t = s_t dS_t K_t,   dK_t = s_t dS_t^T Q_t
//
// B200 mapping (one CTA per SM, persistent, units handed out dynamically):
//   work unit   (bh, 128-key tile); inner loop over 64-query steps that see it
//   warp 0      TMA producer: K1/K2 tile per unit; Q1/Q2 tile + per-row record
//               (LSE1, LSE2, L, s*dL) per step into a 2-stage ring; also
//               fetches the next unit index and publishes it to the other roles
//   warp 1      TMEM owner; issues the contractions of each step:
//                 dK_t += dS_t^T Q_t                        (M=128 keys, N=d_t)
//                 dQ_t^T = K_t^T dS_t^T                     (M=d_t, N=64 queries)
//   warp 14     issues S1^T = K1 Q1^T, S2^T = K2 Q2^T of each step (M=128 keys,
//               N=64) as soon as the query tile is in and the dS warps have read
//               the previous S out, so the tensor pipe works on S of step t+1
//               while dS of step t is formed and while warp 1 waits.
//   warps 2..9  two dS warpgroups, each for 32 of the 64 queries of a step:
//               thread j owns key j (TMEM lane j), loads its S1^T and S2^T
//               row segments, regenerates P1, P2 with exp2 on the MUFU pipe
//               (packed f32x2 arithmetic elsewhere), forms s1*dS1 and s2*dS2
//               in bf16 and writes them once to shared memory in the
//               128B-swizzled layout that serves both as the K-major A operand
//               of dK and the MN-major B operand of dQ^T.  Two warpgroups put
//               two dS warps on every SM sub-partition.
//   warps 10..13 dQ warpgroup: reads dQ^T (thread = feature index) and adds it
//               into the fp32 workspace with coalesced reductions; at the end
//               of a unit converts the dK accumulators to bf16 and stores them.
// TMEM (512 columns): S1^T [0,64) S2^T [64,128) dK1 [128,128+d1) dK2 [..,+d2)
//                     dQ1^T [384,448) dQ2^T [448,512).
//
// Gradient sets (the page's two configurations, same section): the kernel is
// instantiated for SEL = 1 (teacher side only: dQ1, dK1 -- Configuration 2,
// P2 fixed), SEL = 2 (student side only: dQ2, dK2 -- Configuration 1, P1
// fixed, standard distillation) and SEL = 3 (both).  A one-sided instance
// forms, stores and contracts only its own dS, keeps a dQ accumulator of that
// side's width only, and for SEL = 1 skips the P2 exponential (dS1 needs the
// student only through its log-probability, which is linear in S2).  Both S
// products are recomputed in every configuration.
#include "kernels.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

#include <cmath>

namespace skl {
namespace {

constexpr int BK = kBwdBK;  // keys per unit
constexpr int BQ = kBwdBQ;  // queries per step
constexpr int NDS = 2;          // dS warpgroups per CTA
constexpr int QPW = BQ / NDS;   // queries of a step per dS warpgroup
constexpr int DQ_WARP0 = 2 + 4 * NDS;
constexpr int S_WARP = DQ_WARP0 + 4;  // issues the S^T products
constexpr int NTHREADS = (S_WARP + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kColS1 = 0, kColS2 = 64, kColDK1 = 128, kColDQ1 = 384, kColDQ2 = 448;

template <int D1, int D2, int NDT>
struct BwdLayout {  // NDT: dS tiles per buffer (1 or 2 gradient sides)
  static constexpr int k1_bytes = BK * D1 * 2;
  static constexpr int k2_bytes = BK * D2 * 2;
  static constexpr int q1_bytes = BQ * D1 * 2;
  static constexpr int q2_bytes = BQ * D2 * 2;
  static constexpr int rr_bytes = BQ * kRowRec * 4;
  static constexpr int qstage_bytes = q1_bytes + q2_bytes + rr_bytes;
  static constexpr int ds_bytes = BK * BQ * 2;  // one dS^T tile, bf16 [128 keys][64 queries]
  // Deepest Q ring (then most dS buffers) that fits: the Q tile of step t+2
  // must be in flight while step t is contracted.
  static constexpr int fixed_bytes = k1_bytes + k2_bytes + 1024 + 512;
  static constexpr bool fits(int q, int d) {
    return fixed_bytes + q * qstage_bytes + d * NDT * ds_bytes <= 232448;
  }
  static constexpr int QSTAGES = fits(4, 2) ? 4 : (fits(3, 2) ? 3 : (fits(4, 1) ? 4 : 3));
  static constexpr int DSBUF = fits(QSTAGES, 2) ? 2 : 1;
  static constexpr int k1_off = 0;
  static constexpr int k2_off = k1_off + k1_bytes;
  static constexpr int q_off = k2_off + k2_bytes;
  static constexpr int ds_off = q_off + QSTAGES * qstage_bytes;
  static constexpr int bar_off = ds_off + DSBUF * NDT * ds_bytes;
  // kfull kempty qfull[Q] qempty[Q] sfull sempty dsfull[D] dsempty[D] dqfull dqempty1
  // dqempty2 dkfull dkempty ufull[2] uempty[2] drain
  static constexpr int nbar = 2 + 2 * QSTAGES + 2 + 2 * DSBUF + 5 + 4 + 1;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int total = misc_off + 32;
  static constexpr int alloc = total + 1024;
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(k1_bytes % 1024 == 0 && k2_bytes % 1024 == 0 && q1_bytes % 1024 == 0 &&
                    q2_bytes % 1024 == 0 && rr_bytes % 1024 == 0,
                "operand tiles must stay 1024-byte aligned");
};

struct UnitB {
  int bh, k0, qt0, nsteps, rot;
  // Query tile of step t (steps may start at a rotation rot; the sums over
  // query tiles do not depend on the order).
  __device__ __forceinline__ int qt(int t) const {
    int r = t + rot;
    if (r >= nsteps) r -= nsteps;
    return qt0 + r;
  }
};

__device__ __forceinline__ UnitB decode_unit(const BwdParams& p, int u) {
  const int nkt = (p.NK + BK - 1) / BK;
  UnitB w;
  w.bh = u / nkt;  // head-major: few heads active at once keeps Q and dQacc in L2
  const int kt = u % nkt;  // within a head, the key tiles with the most query steps first
  w.k0 = kt * BK;
  const int nqt = p.NQpad / BQ;
  int qt0 = 0;
  if (p.causal) {
    const int first = w.k0 - (p.NK - p.NQ);  // first query row that sees key k0
    qt0 = first > 0 ? first / BQ : 0;
  }
  w.qt0 = qt0;
  w.nsteps = nqt - qt0;
  w.rot = 0;
  return w;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// dS for one key row and QPW queries of a step (pairs of queries at a time,
// packed f32x2).  s1/s2: raw products <K_t[key], Q_t[q]> from TMEM; rr: the
// step's field-major row records offset to this half; w1/w2 receive the bf16
// pairs of s1*dS1^T and s2*dS2^T for these queries.  EARLY: also store each
// 8-query chunk into row j of the dS tiles as soon as it is formed, so that
// the stores overlap the arithmetic (the buffer must already be free).
//   u_t = log2 P_t = c_t S_t - LSE_t log2e
//   dS1 = s1 dL P1 (ln2 (u1 - u2) - L),   dS2 = s2 dL (P2 - P1)
// MASK: visible iff key < NK and (not causal or q >= thr), with thr the first
// visible query index of this half for this key.
template <bool MASK, bool G1, bool G2, bool EARLY = false>
__device__ __forceinline__ void form_ds(const uint32_t (&s1)[QPW], const uint32_t (&s2)[QPW],
                                        const float* rr, float c1, float c2, bool key_ok, int thr,
                                        uint32_t (&w1)[QPW / 2], uint32_t (&w2)[QPW / 2],
                                        int j = 0, int c0 = 0, uint32_t ds1_row = 0,
                                        uint32_t ds2_row = 0) {
  const float2 C1 = make_float2(c1, c1), C2 = make_float2(c2, c2);
  const float2 NEG1 = make_float2(-1.f, -1.f), LN2 = make_float2(kLn2, kLn2);
#pragma unroll
  for (int c = 0; c < QPW / 8; ++c) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {  // 4 queries per h
      const int q = c * 8 + h * 4;
      const float4 nb1 = ld_shared_f4(rr + 0 * BQ + q);
      const float4 nb2 = ld_shared_f4(rr + 1 * BQ + q);
      const float4 nL = ld_shared_f4(rr + 2 * BQ + q);
      const float4 g1 = G1 ? ld_shared_f4(rr + 3 * BQ + q) : float4{};
      const float4 g2 = G2 ? ld_shared_f4(rr + 4 * BQ + q) : float4{};
#pragma unroll
      for (int e = 0; e < 2; ++e) {  // a pair of queries
        const int i = q + 2 * e;
        const float2 S1 = make_float2(__uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
        const float2 S2 = make_float2(__uint_as_float(s2[i]), __uint_as_float(s2[i + 1]));
        const float2 B1 = e ? make_float2(nb1.z, nb1.w) : make_float2(nb1.x, nb1.y);
        const float2 B2 = e ? make_float2(nb2.z, nb2.w) : make_float2(nb2.x, nb2.y);
        const float2 NL = e ? make_float2(nL.z, nL.w) : make_float2(nL.x, nL.y);
        const float2 Gs1 = e ? make_float2(g1.z, g1.w) : make_float2(g1.x, g1.y);
        const float2 Gs2 = e ? make_float2(g2.z, g2.w) : make_float2(g2.x, g2.y);
        const float2 u1 = __ffma2_rn(S1, C1, B1);
        const float2 u2 = __ffma2_rn(S2, C2, B2);
        const float2 P1 = make_float2(ex2(u1.x), ex2(u1.y));
        float2 d1 = make_float2(0.f, 0.f), d2 = make_float2(0.f, 0.f);
        if (G1) {
          const float2 t = __ffma2_rn(__ffma2_rn(u2, NEG1, u1), LN2, NL);
          d1 = __fmul2_rn(__fmul2_rn(P1, t), Gs1);
        }
        if (G2) {
          const float2 P2 = make_float2(ex2(u2.x), ex2(u2.y));
          d2 = __fmul2_rn(__ffma2_rn(P1, NEG1, P2), Gs2);
        }
        if (MASK) {
          const bool vx = key_ok && i >= thr, vy = key_ok && i + 1 >= thr;
          d1.x = vx ? d1.x : 0.f;
          d2.x = vx ? d2.x : 0.f;
          d1.y = vy ? d1.y : 0.f;
          d2.y = vy ? d2.y : 0.f;
        }
        if (G1) w1[c * 4 + h * 2 + e] = pack_bf16(d1.x, d1.y);
        if (G2) w2[c * 4 + h * 2 + e] = pack_bf16(d2.x, d2.y);
      }
    }
    if (EARLY) {  // this 8-query chunk goes to shared memory at once (swizzle as in store_ds)
      const uint32_t sw = static_cast<uint32_t>(((c0 + c) ^ (j & 7)) << 4);
      if (G1) st_shared_v4(ds1_row + sw, w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
      if (G2) st_shared_v4(ds2_row + sw, w2[4 * c], w2[4 * c + 1], w2[4 * c + 2], w2[4 * c + 3]);
    }
  }
}

// Stores the packed dS row segments of one key into the 128B-swizzled tiles:
// 16-byte chunk c0 + c of row j lands at chunk (c0 + c) ^ (j mod 8).
template <bool G1, bool G2>
__device__ __forceinline__ void store_ds(const uint32_t (&w1)[QPW / 2],
                                         const uint32_t (&w2)[QPW / 2], int j, int c0,
                                         uint32_t ds1_row, uint32_t ds2_row) {
#pragma unroll
  for (int c = 0; c < QPW / 8; ++c) {
    const uint32_t sw = static_cast<uint32_t>(((c0 + c) ^ (j & 7)) << 4);
    if (G1) st_shared_v4(ds1_row + sw, w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
    if (G2) st_shared_v4(ds2_row + sw, w2[4 * c], w2[4 * c + 1], w2[4 * c + 2], w2[4 * c + 3]);
  }
}

// Adds 32 queries of one dQ_t^T feature row into the fp32 accumulator: base
// points at the first query's row, feature f; rows are LDQ floats apart.
template <int LDQ, bool FULL>
__device__ __forceinline__ void red_dq(float* base, const uint32_t (&v)[32], int nvalid) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (FULL || i < nvalid) atomicAdd(base + i * LDQ, __uint_as_float(v[i]));
}

template <int D1, int D2, int SEL>
__global__ void __launch_bounds__(NTHREADS, 1) streamkl_bwd_kernel(const __grid_constant__ BwdParams p) {
  constexpr bool G1 = (SEL & 1) != 0, G2 = (SEL & 2) != 0;
  using Lay = BwdLayout<D1, D2, (G1 ? 1 : 0) + (G2 ? 1 : 0)>;
  constexpr int QST = Lay::QSTAGES;
  constexpr int DSB = Lay::DSBUF;
  // dQ accumulator row: the wanted sides only, teacher first
  constexpr int LDQ = (G1 ? D1 : 0) + (G2 ? D2 : 0);
  constexpr int DQ2_COL = G1 ? D1 : 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* kfull = bars + 0;
  uint64_t* kempty = bars + 1;
  uint64_t* qfull = bars + 2;
  uint64_t* qempty = qfull + QST;
  uint64_t* sfull = qempty + QST;
  uint64_t* sempty = sfull + 1;
  uint64_t* dsfull = sempty + 1;
  uint64_t* dsempty = dsfull + DSB;
  uint64_t* dqfull = dsempty + DSB;
  uint64_t* dqempty = dqfull + 1;  // [2]: dQ1^T and dQ2^T slots read out
  uint64_t* dkfull = dqempty + 2;
  uint64_t* dkempty = dkfull + 1;
  uint64_t* ufull = dkempty + 1;
  uint64_t* uempty = ufull + 2;
  uint64_t* drain = uempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 4);
  volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 8);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(kfull, 1);
    mbar_init(kempty, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(&qfull[s], 1);
      mbar_init(&qempty[s], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(sempty, 4 * NDS);  // every warp of every dS warpgroup
    for (int s = 0; s < DSB; ++s) {
      mbar_init(&dsfull[s], 4 * NDS);
      mbar_init(&dsempty[s], 1);
    }
    mbar_init(dqfull, 1);
    mbar_init(&dqempty[0], 4);
    mbar_init(&dqempty[1], 4);
    mbar_init(dkfull, 1);
    mbar_init(dkempty, 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ufull[s], 1);
      mbar_init(&uempty[s], 2 + 4 * NDS + 4);  // both UMMA issuers + dS warps + dQ warps
    }
    mbar_init(drain, 2);
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

  const int nkt = (p.NK + BK - 1) / BK;
  const int total = p.BH * nkt;
  int* counter = reinterpret_cast<int*>(const_cast<float*>(p.rowrec) +
                                        static_cast<size_t>(p.BH) * p.NQpad * kRowRec);
  uint8_t* k1_s = smem + Lay::k1_off;
  uint8_t* k2_s = smem + Lay::k2_off;
  auto q1_s = [&](int s) { return smem + Lay::q_off + s * Lay::qstage_bytes; };
  auto q2_s = [&](int s) { return smem + Lay::q_off + s * Lay::qstage_bytes + Lay::q1_bytes; };
  auto rr_s = [&](int s) {
    return reinterpret_cast<float*>(smem + Lay::q_off + s * Lay::qstage_bytes + Lay::q1_bytes +
                                    Lay::q2_bytes);
  };
  constexpr int NDT = (G1 ? 1 : 0) + (G2 ? 1 : 0);
  auto ds1_s = [&](int b) { return smem + Lay::ds_off + b * NDT * Lay::ds_bytes; };
  auto ds2_s = [&](int b) {
    return smem + Lay::ds_off + b * NDT * Lay::ds_bytes + (G1 ? Lay::ds_bytes : 0);
  };
  const int off = p.NK - p.NQ;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int us = 0, qs = 0;
      uint32_t uph = 0, kph = 0, qph = 0;
      uint32_t armed_k = 0, armed_q[QST] = {};
      int next = blockIdx.x;
      bool ok = true;
      for (;;) {
        const int u = next < total ? next : -1;
        if (!(ok = mbar_wait(&uempty[us], uph ^ 1, ctl))) break;
        unit_slot[us] = u;
        mbar_arrive(&ufull[us]);
        if (++us == 2) {
          us = 0;
          uph ^= 1;
        }
        if (u < 0) break;
        const UnitB w = decode_unit(p, u);
        if (!(ok = mbar_wait(kempty, kph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(kfull, Lay::k1_bytes + Lay::k2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(k1_s + b * (BK * 128), &p.tmK1, kfull, b * 64, w.k0, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(k2_s + b * (BK * 128), &p.tmK2, kfull, b * 64, w.k0, w.bh);
        armed_k = kph + 1;
        kph ^= 1;
        for (int t = 0; t < w.nsteps; ++t) {
          const int q0 = w.qt(t) * BQ;
          if (!(ok = mbar_wait(&qempty[qs], qph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&qfull[qs], Lay::qstage_bytes);
#pragma unroll
          for (int b = 0; b < D1 / 64; ++b)
            tma_load_3d(q1_s(qs) + b * (BQ * 128), &p.tmQ1, &qfull[qs], b * 64, q0, w.bh);
#pragma unroll
          for (int b = 0; b < D2 / 64; ++b)
            tma_load_3d(q2_s(qs) + b * (BQ * 128), &p.tmQ2, &qfull[qs], b * 64, q0, w.bh);
          bulk_load(rr_s(qs), p.rowrec + (static_cast<size_t>(w.bh) * p.NQpad + q0) * kRowRec,
                    Lay::rr_bytes, &qfull[qs]);
          armed_q[qs] = qph + 1;
          if (++qs == QST) {
            qs = 0;
            qph ^= 1;
          }
        }
        if (!ok) break;
        next = static_cast<int>(gridDim.x) + atomicAdd(counter, 1);
      }
      if (!ok) {
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        if (armed_k) mbar_wait(kfull, armed_k - 1, dctl);
        for (int s = 0; s < QST; ++s)
          if (armed_q[s]) mbar_wait(&qfull[s], armed_q[s] - 1, dctl);
      }
    }
  } else if (warp == 1 || warp == S_WARP) {
    // ------------------------------------------------------------ UMMA issuers
    // The S^T products come from warp S_WARP, the contractions from warp 1 (the
    // queue in front of the tensor pipe holds about one product, so one
    // stream's barrier waits are filled by the other's products).  Each commit
    // tracks its own thread's products; the contractions of a step imply its
    // S^T (their dS was formed from it), so the stage and unit releases below
    // stay with warp 1.
    if (lane == 0) {
      const bool s_role = warp == S_WARP;
      constexpr uint32_t idS = idesc_bf16(BK, BQ);                // S^T: M=128 keys, N=64
      constexpr uint32_t idK1 = idesc_bf16(BK, D1, 0, 1);         // dK1: B = Q1 MN-major
      constexpr uint32_t idK2 = idesc_bf16(BK, D2, 0, 1);
      constexpr uint32_t idQ1 = idesc_bf16(D1, BQ, 1, 1);         // dQ1^T: A = K1 MN-major
      constexpr uint32_t idQ2 = idesc_bf16(D2, BQ, 1, 1);
      const uint32_t k1a = smem_u32(k1_s), k2a = smem_u32(k2_s);
      const uint64_t k1d = sdesc_sw128(k1a, 16, 1024), k2d = sdesc_sw128(k2a, 16, 1024);
      // K tiles read MN-major for dQ^T: 64-feature chunks 16 KB apart
      const uint64_t k1m = sdesc_sw128(k1a, BK * 128, 1024), k2m = sdesc_sw128(k2a, BK * 128, 1024);
      int us = 0, qs_s = 0, qs_r = 0, db = 0;
      uint32_t uph = 0, kph = 0, qph_s = 0, sph = 0, dkph = 0;
      uint32_t dqph[2] = {0, 0};
      uint32_t dsph[DSB] = {};
      bool ok = true;
      for (;;) {
        if (!(ok = mbar_wait(&ufull[us], uph, ctl))) break;
        const int u = unit_slot[us];
        mbar_arrive(&uempty[us]);
        if (++us == 2) {
          us = 0;
          uph ^= 1;
        }
        if (u < 0) break;
        const UnitB w = decode_unit(p, u);
        if (s_role) {
          if (!(ok = mbar_wait(kfull, kph, ctl))) break;
          kph ^= 1;
        }
        auto issue_s = [&]() -> bool {
          if (!mbar_wait(&qfull[qs_s], qph_s, ctl)) return false;
          if (!mbar_wait(sempty, sph ^ 1, ctl)) return false;
          tc_fence_after();
          const uint64_t q1d = sdesc_sw128(smem_u32(q1_s(qs_s)), 16, 1024);
          const uint64_t q2d = sdesc_sw128(smem_u32(q2_s(qs_s)), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D1 / 16; ++kk) {
            const uint32_t o = (kk & 3) * 32;
            umma_bf16_ss(tmem_base + kColS1, sdesc_advance(k1d, (kk >> 2) * (BK * 128) + o),
                         sdesc_advance(q1d, (kk >> 2) * (BQ * 128) + o), idS, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D2 / 16; ++kk) {
            const uint32_t o = (kk & 3) * 32;
            umma_bf16_ss(tmem_base + kColS2, sdesc_advance(k2d, (kk >> 2) * (BK * 128) + o),
                         sdesc_advance(q2d, (kk >> 2) * (BQ * 128) + o), idS, kk > 0);
          }
          umma_commit(sfull);
          sph ^= 1;
          if (++qs_s == QST) {
            qs_s = 0;
            qph_s ^= 1;
          }
          return true;
        };
        if (s_role) {
          for (int t = 0; t < w.nsteps && ok; ++t) ok = issue_s();
          if (!ok) break;
          continue;
        }
        for (int t = 0; t < w.nsteps && ok; ++t) {
          if (!(ok = mbar_wait(&dsfull[db], dsph[db], ctl))) break;
          dsph[db] ^= 1;
          if (t == 0) {
            if (!(ok = mbar_wait(dkempty, dkph ^ 1, ctl))) break;
            dkph ^= 1;
          }
          tc_fence_after();
          // dS^T tiles read K-major for dK and MN-major for dQ^T; Q tiles MN-major for dK
          const uint64_t q1m = sdesc_sw128(smem_u32(q1_s(qs_r)), BQ * 128, 1024);
          const uint64_t q2m = sdesc_sw128(smem_u32(q2_s(qs_r)), BQ * 128, 1024);
          const uint64_t d1k = sdesc_sw128(smem_u32(ds1_s(db)), 16, 1024);
          const uint64_t d2k = sdesc_sw128(smem_u32(ds2_s(db)), 16, 1024);
          const uint64_t d1m = sdesc_sw128(smem_u32(ds1_s(db)), BQ * 128, 1024);
          const uint64_t d2m = sdesc_sw128(smem_u32(ds2_s(db)), BQ * 128, 1024);
          // dK_t += (s_t dS_t)^T Q_t : A = dS^T (K-major, 128B rows of 64 queries),
          // B = Q_t read MN-major (features contiguous; 64-feature chunks 8 KB apart).
#pragma unroll
          for (int kk = 0; kk < BQ / 16; ++kk) {
            if (G1 && p.want_dk1)
              umma_bf16_ss(tmem_base + kColDK1, sdesc_sw128(smem_u32(ds1_s(db)) + kk * 32, 16, 1024),
                           sdesc_sw128(smem_u32(q1_s(qs_r)) + kk * 2048, BQ * 128, 1024), idK1, (t > 0 || kk > 0));
            if (G2 && p.want_dk2)
              umma_bf16_ss(tmem_base + kColDK1 + D1, sdesc_sw128(smem_u32(ds2_s(db)) + kk * 32, 16, 1024),
                           sdesc_sw128(smem_u32(q2_s(qs_r)) + kk * 2048, BQ * 128, 1024), idK2, (t > 0 || kk > 0));
          }
          // dQ_t^T = K_t^T (s_t dS_t)^T : A = K tile read MN-major (64-feature chunks
          // 16 KB apart), B = dS^T read MN-major (64 queries contiguous per key).
          if (G1) {
            if (!(ok = mbar_wait(&dqempty[0], dqph[0] ^ 1, ctl))) break;
            dqph[0] ^= 1;
            tc_fence_after();
            if (p.want_dq1) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16_ss(tmem_base + kColDQ1, sdesc_advance(k1m, kk * 2048),
                             sdesc_advance(d1m, kk * 2048), idQ1, kk > 0);
            }
          }
          if (G2) {
            if (!(ok = mbar_wait(&dqempty[1], dqph[1] ^ 1, ctl))) break;
            dqph[1] ^= 1;
            tc_fence_after();
            if (p.want_dq2) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma_bf16_ss(tmem_base + kColDQ2, sdesc_advance(k2m, kk * 2048),
                             sdesc_advance(d2m, kk * 2048), idQ2, kk > 0);
            }
          }
          umma_commit(dqfull);
          umma_commit(&dsempty[db]);
          umma_commit(&qempty[qs_r]);
          if (++db == DSB) db = 0;
          if (++qs_r == QST) qs_r = 0;
        }
        if (!ok) break;
        umma_commit(dkfull);
        umma_commit(kempty);
      }
      // Every product of both issuers is complete before TMEM is released: drain
      // counts a commit from each, and warp 1, which releases TMEM after the
      // final barrier, waits for it.  The S issuer, which may finish a unit
      // ahead, does not wait (its wait would span warp 1's whole last unit).
      umma_commit(drain);
      if (!s_role) {
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        mbar_wait(drain, 0, dctl);
      }
    }
  } else if (warp < DQ_WARP0) {
    // ------------------------------------------------------------ dS warpgroups
    const int part = (warp - 2) >> 2;  // queries [part*QPW, part*QPW + QPW) of each step
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // key row within the tile
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int us = 0, qs = 0, db = 0;
    uint32_t uph = 0, qph = 0, sph = 0;
    uint32_t dsph[DSB] = {};
    bool ok = true;
    for (;;) {
      if (!(ok = mbar_wait(&ufull[us], uph, ctl))) break;
      const int u = unit_slot[us];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[us]);
      if (++us == 2) {
        us = 0;
        uph ^= 1;
      }
      if (u < 0) break;
      const UnitB w = decode_unit(p, u);
      const int key = w.k0 + j;
      const bool key_ok = key < p.NK;
      for (int t = 0; t < w.nsteps; ++t) {
        const int q0 = w.qt(t) * BQ;
        if (!(ok = mbar_wait(&qfull[qs], qph, ctl))) break;  // row records of this step
        if (!(ok = mbar_wait(sfull, sph, ctl))) break;
        sph ^= 1;
        tc_fence_after();
        uint32_t a[QPW], b[QPW];
        tmem_ld_32x32b<QPW>(tl + kColS1 + part * QPW, a);
        tmem_ld_32x32b<QPW>(tl + kColS2 + part * QPW, b);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(sempty);
        const float* rr = rr_s(qs) + part * QPW;
        const bool masked = (p.causal && q0 + off < w.k0 + BK - 1) || (w.k0 + BK > p.NK);
        uint32_t w1[QPW / 2], w2[QPW / 2];
        const int thr = p.causal ? key - off - q0 - part * QPW : -1;  // first visible query
        const uint32_t r1 = smem_u32(ds1_s(db)) + j * 128, r2 = smem_u32(ds2_s(db)) + j * 128;
        if (DSB >= 2) {
          // With two dS buffers the one this step writes was freed a step ago:
          // wait for it first and store as the chunks are formed.
          if (!(ok = mbar_wait(&dsempty[db], dsph[db] ^ 1, ctl))) break;
          dsph[db] ^= 1;
          if (masked)
            form_ds<true, G1, G2, true>(a, b, rr, p.c1, p.c2, key_ok, thr, w1, w2, j,
                                        part * (QPW / 8), r1, r2);
          else
            form_ds<false, G1, G2, true>(a, b, rr, p.c1, p.c2, true, 0, w1, w2, j,
                                         part * (QPW / 8), r1, r2);
        } else {
          // One buffer: form dS in registers while the previous step's
          // contractions still read it.
          if (masked)
            form_ds<true, G1, G2>(a, b, rr, p.c1, p.c2, key_ok, thr, w1, w2);
          else
            form_ds<false, G1, G2>(a, b, rr, p.c1, p.c2, true, 0, w1, w2);
          // the buffer is free once the contractions of the step that used it are done
          if (!(ok = mbar_wait(&dsempty[db], dsph[db] ^ 1, ctl))) break;
          dsph[db] ^= 1;
          store_ds<G1, G2>(w1, w2, j, part * (QPW / 8), r1, r2);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dsfull[db]);
        if (++db == DSB) db = 0;
        if (++qs == QST) {
          qs = 0;
          qph ^= 1;
        }
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ dQ / dK warpgroup
    const int quarter = warp & 3;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    // dQ_t^T rows are features: M = 128 puts feature f in lane f; M = 64 puts
    // features 16q..16q+15 in lanes 32q..32q+15.
    const int f1 = (D1 == 128) ? quarter * 32 + lane : (lane < 16 ? quarter * 16 + lane : -1);
    const int f2 = (D2 == 128) ? quarter * 32 + lane : (lane < 16 ? quarter * 16 + lane : -1);
    int us = 0;
    uint32_t uph = 0, dqph = 0, dkph = 0;
    bool ok = true;
    for (;;) {
      if (!(ok = mbar_wait(&ufull[us], uph, ctl))) break;
      const int u = unit_slot[us];
      __syncwarp();
      if (lane == 0) mbar_arrive(&uempty[us]);
      if (++us == 2) {
        us = 0;
        uph ^= 1;
      }
      if (u < 0) break;
      const UnitB w = decode_unit(p, u);
      for (int t = 0; t < w.nsteps; ++t) {
        const int q0 = w.qt(t) * BQ;
        if (!(ok = mbar_wait(dqfull, dqph, ctl))) break;
        dqph ^= 1;
        tc_fence_after();
        const int nvalid = min(BQ, p.NQ - q0);
        float* base = p.dQacc + (static_cast<size_t>(w.bh) * p.NQ + q0) * LDQ;
#pragma unroll
        for (int tsel = 0; tsel < 2; ++tsel) {
          if ((tsel == 0 && !G1) || (tsel == 1 && !G2)) continue;
          const bool want = tsel == 0 ? p.want_dq1 : p.want_dq2;
          const int f = tsel == 0 ? f1 : DQ2_COL + f2;
          const bool fok = (tsel == 0 ? f1 : f2) >= 0;
          const uint32_t col = tl + (tsel == 0 ? kColDQ1 : kColDQ2);
          // two halves of 32 queries; the slot is released once both are in registers
          uint32_t v0[32], v1[32];
          if (want) {
            tmem_ld_32x32b_x32(col, v0);
            tmem_ld_wait();
            reg_fence(v0);
          }
          if (want && fok) {
            if (nvalid == BQ)
              red_dq<LDQ, true>(base + f, v0, 32);
            else
              red_dq<LDQ, false>(base + f, v0, nvalid);
          }
          if (want) {
            tmem_ld_32x32b_x32(col + 32, v1);
            tmem_ld_wait();
            reg_fence(v1);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dqempty[tsel]);
          if (want && fok) {
            if (nvalid == BQ)
              red_dq<LDQ, true>(base + 32 * LDQ + f, v1, 32);
            else
              red_dq<LDQ, false>(base + 32 * LDQ + f, v1, nvalid - 32);
          }
        }
      }
      if (!ok) break;
      // Unit epilogue: dK accumulators (thread = key row) to bf16.
      if (!(ok = mbar_wait(dkfull, dkph, ctl))) break;
      dkph ^= 1;
      tc_fence_after();
      const int key = w.k0 + quarter * 32 + lane;
      const bool row_ok = key < p.NK;
#pragma unroll
      for (int tsel = 0; tsel < 2; ++tsel) {
        if ((tsel == 0 && !G1) || (tsel == 1 && !G2)) continue;
        const bool want = tsel == 0 ? p.want_dk1 : p.want_dk2;
        if (!want) continue;
        constexpr int DMAX = D1 > D2 ? D1 : D2;
        const int D = tsel == 0 ? D1 : D2;
        __nv_bfloat16* dst =
            (tsel == 0 ? p.dK1 : p.dK2) + (static_cast<size_t>(w.bh) * p.NK + key) * D;
        const uint32_t col0 = tl + kColDK1 + (tsel == 0 ? 0 : D1);
#pragma unroll
        for (int c = 0; c < DMAX; c += 32) {
          if (c >= D) break;
          uint32_t v[32];
          tmem_ld_32x32b_x32(col0 + c, v);
          tmem_ld_wait();
          reg_fence(v);
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 32; e += 8) {
              uint4 o;
              o.x = pack_bf16(__uint_as_float(v[e + 0]), __uint_as_float(v[e + 1]));
              o.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
              o.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
              o.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
              *reinterpret_cast<uint4*>(dst + c + e) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkempty);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// Per-row records for the key-tile backward, field-major per 64-row step
// ([bh][step][field][64]): -LSE1*log2e, -LSE2*log2e, -L, s1*dL, s2*dL, 0, 0, 0.
// Rows past NQ (padding of the last step) get all zeros, so their weight is
// zero and they contribute nothing.  Without a record buffer (the query-tile
// kernel) only the zeroing is done.  Also zeroes the fp32 accumulator and the
// two work-unit counters.
__global__ void streamkl_bwd_prep_kernel(const BwdPrepParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long nrec = p.rowrec ? static_cast<long long>(p.BH) * p.NQpad : 0;
  constexpr float kLog2e = 1.4426950408889634f;
  constexpr int S = kBwdBQ;
  for (long long r = tid; r < nrec; r += stride) {
    const int bh = static_cast<int>(r / p.NQpad);
    const int i = static_cast<int>(r % p.NQpad);
    float f[kRowRec] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (i < p.NQ) {
      const size_t o = static_cast<size_t>(bh) * p.NQ + i;
      const float g = p.dL[o];
      f[0] = -p.LSE1[o] * kLog2e;
      f[1] = -p.LSE2[o] * kLog2e;
      f[2] = -p.L[o];
      f[3] = p.s1 * g;
      f[4] = p.s2 * g;
    }
    float* rec = p.rowrec + (static_cast<size_t>(bh) * p.NQpad + (i / S) * S) * kRowRec + (i % S);
#pragma unroll
    for (int k = 0; k < kRowRec; ++k) rec[k * S] = f[k];
  }
  const long long n4 = p.dqacc_elems / 4;
  for (long long e = tid; e < n4; e += stride)
    reinterpret_cast<float4*>(p.dQacc)[e] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (tid == 0) {
    p.counters[0] = 0;
    p.counters[1] = 0;
  }
}

// fp32 dQ accumulator [rows][d1 + d2] -> bf16 dQ1 [rows][d1], dQ2 [rows][d2].
__global__ void streamkl_bwd_convert_kernel(const BwdConvertParams p) {
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  const int ld = p.d1 + p.d2;
  const long long chunks = p.rows * (ld / 8);
  for (long long c = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; c < chunks;
       c += stride) {
    const long long r = c / (ld / 8);
    const int col = static_cast<int>(c % (ld / 8)) * 8;
    const float4* src = reinterpret_cast<const float4*>(p.dQacc + r * ld + col);
    const float4 x = src[0], y = src[1];
    uint4 o;
    o.x = pack_bf16(x.x, x.y);
    o.y = pack_bf16(x.z, x.w);
    o.z = pack_bf16(y.x, y.y);
    o.w = pack_bf16(y.z, y.w);
    if (col < p.d1) {
      if (p.dQ1) *reinterpret_cast<uint4*>(p.dQ1 + r * p.d1 + col) = o;
    } else {
      if (p.dQ2) *reinterpret_cast<uint4*>(p.dQ2 + r * p.d2 + (col - p.d1)) = o;
    }
  }
}

template <int D1, int D2, int SEL>
cudaError_t launch_t(const BwdParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = BwdLayout<D1, D2, (SEL == 3) ? 2 : 1>::alloc;
  auto kern = streamkl_bwd_kernel<D1, D2, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_smem_bytes(int d1, int d2) {
  if (d1 == 128 && d2 == 128) return BwdLayout<128, 128, 2>::alloc;
  if (d1 == 128 && d2 == 64) return BwdLayout<128, 64, 2>::alloc;
  if (d1 == 64 && d2 == 128) return BwdLayout<64, 128, 2>::alloc;
  if (d1 == 64 && d2 == 64) return BwdLayout<64, 64, 2>::alloc;
  return 0;
}

template <int SEL>
cudaError_t launch_sel(const BwdParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128, SEL>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64, SEL>(p, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd(const BwdParams& p, int d1, int d2, int sel, int grid, cudaStream_t stream) {
  if (sel == 1) return launch_sel<1>(p, d1, d2, grid, stream);
  if (sel == 2) return launch_sel<2>(p, d1, d2, grid, stream);
  if (sel == 3) return launch_sel<3>(p, d1, d2, grid, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_prep(const BwdPrepParams& p, int num_sms, cudaStream_t stream) {
  streamkl_bwd_prep_kernel<<<num_sms * 4, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_bwd_convert(const BwdConvertParams& p, int num_sms, cudaStream_t stream) {
  streamkl_bwd_convert_kernel<<<num_sms * 4, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace skl
