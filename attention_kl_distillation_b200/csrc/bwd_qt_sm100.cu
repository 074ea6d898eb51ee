// bwd_qt_sm100.cu -- recompute backward of the fused attention-KL for sm_100a,
// query-tile variant.
//
// Same arithmetic as bwd_sm100.cu (StreamKL summary page, "Metodologia"
// section 2: P_t = exp(x_t - LSE_t) regenerated tile by tile from the saved
// vectors, every visible (query, key) pair visited once, one of the two
// gradients accumulated with atomics), with the roles of queries and keys
// exchanged:
//
//   dS1 = g * P1 * ((x1 - LSE1) - (x2 - LSE2) - L),   dS2 = g * (P2 - P1)
//   dQ_t = s_t dS_t K_t   (on chip, over the unit's key steps)
//   dK_t = s_t dS_t^T Q_t (fp32 reductions into the workspace, over query tiles)
//
// Why this orientation: a thread of the dS warps owns one query row (one TMEM
// lane), so the per-query quantities dS needs (LSE1, LSE2, L, dL) are a few
// registers loaded once per unit.  In the key-tile kernel a thread owns a key
// and reads them from shared memory for every query of every step, which is
// close to a third of the shared-memory traffic that bounds that kernel.  The
// key-tile kernel stays the choice when there are few query tiles to spread
// over the SMs.
//
// B200 mapping (one CTA per SM, persistent, units handed out dynamically):
//   work unit   (bh, 128-query tile); inner loop over the 64-key steps it sees
//   warp 0      TMA producer: Q1/Q2 tile per unit, K1/K2 tiles per step into
//               a ring; fetches the next unit index and publishes it
//   warp 1      TMEM owner; issues the contractions of each step:
//                 dQ_t += dS_t K_t                          (M=128 queries, N=d_t)
//                 dK_t^T = Q_t^T dS_t                       (M=d_t, N=64 keys)
//   warp 14     issues S1 = Q1 K1^T, S2 = Q2 K2^T of each step (M=128 queries,
//               N=64), as soon as the key tile is in and the dS warps have read
//               the previous S out; the two issuing threads keep the tensor
//               pipe fed while the other waits on a barrier.
//   warps 2..9  two dS warpgroups, each for 32 of the 64 keys of a step:
//               thread r owns query row r (TMEM lane r), loads its S1 and S2
//               segments, regenerates P1, P2 (exp2 on the MUFU pipe, packed
//               f32x2 arithmetic elsewhere) and writes s1*dS1 and s2*dS2 in
//               bf16 once to shared memory, in the 128B-swizzled layout that is
//               the K-major A operand of dQ and the MN-major B operand of dK^T.
//   warps 10..13 dK warpgroup: reads dK^T (thread = feature) and adds it into
//               the fp32 workspace with coalesced reductions; at the end of a
//               unit converts the dQ accumulators to bf16 and stores them.
// TMEM (512 columns): S1 [0,64) S2 [64,128) dQ1 [128,128+d1) dQ2 [..,+d2)
//                     dK1^T [384,448) dK2^T [448,512).  A one-sided instance
//                     keeps its side's dQ from column 128 and a second S buffer
//                     after it, so S of step t+1 need not wait for the dS warps
//                     to read S of step t.
//
// Gradient sets as in the key-tile kernel: SEL = 1 (teacher side), 2 (student
// side), 3 (both); a one-sided instance forms and contracts only its own dS,
// reduces a dK accumulator of that side's width only, and SEL = 1 skips the
// P2 exponential.
#include "kernels.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

#include <cmath>

namespace skl {
namespace {

constexpr int RQ = kBwdQtRows;  // queries per unit
constexpr int CK = kBwdQtKeys;  // keys per step
constexpr int NDS = 2;          // dS warpgroups per CTA
constexpr int KPW = CK / NDS;   // keys of a step per dS warpgroup
constexpr int DK_WARP0 = 2 + 4 * NDS;
constexpr int S_WARP = DK_WARP0 + 4;  // issues the S products
constexpr int NTHREADS = (S_WARP + 1) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColS1 = 0, kColS2 = 64, kColDQ1 = 128, kColDK1 = 384, kColDK2 = 448;

template <int D1, int D2, int NDT>
struct QtLayout {  // NDT: dS tiles per buffer (1 or 2 gradient sides)
  static constexpr int q1_bytes = RQ * D1 * 2;
  static constexpr int q2_bytes = RQ * D2 * 2;
  static constexpr int k1_bytes = CK * D1 * 2;
  static constexpr int k2_bytes = CK * D2 * 2;
  static constexpr int kstage_bytes = k1_bytes + k2_bytes;
  static constexpr int ds_bytes = RQ * CK * 2;  // one dS tile, bf16 [128 queries][64 keys]
  // One dS buffer: the dS warps store a step's dS once the previous step's
  // contractions are done with it.  A second buffer (which fits next to a
  // 3-deep key ring) measured slower on B1 H32 N16384 d128 causal, 10.4 against
  // 9.1 ms; the deepest key ring that fits is kept instead (the key tile of
  // step t+2 must be in flight while step t is contracted).
  static constexpr int fixed_bytes = q1_bytes + q2_bytes + 1024 + 512;
  static constexpr bool fits(int k, int d) {
    return fixed_bytes + k * kstage_bytes + d * NDT * ds_bytes <= 232448;
  }
  static constexpr int DSBUF = 1;  // the dS warps' store waits on the previous step's kempty
  static constexpr int KSTAGES = fits(4, DSBUF) ? 4 : 3;
  static constexpr int q1_off = 0;
  static constexpr int q2_off = q1_off + q1_bytes;
  static constexpr int k_off = q2_off + q2_bytes;
  static constexpr int ds_off = k_off + KSTAGES * kstage_bytes;
  static constexpr int bar_off = ds_off + DSBUF * NDT * ds_bytes;
  // qfull qempty kfull[K] kempty[K] sfull[2] sempty[2] dsfull[D] dkempty[2]
  // dqfull dqempty ufull[2] uempty[2] drain
  static constexpr int nbar = 2 + 2 * KSTAGES + 4 + DSBUF + 4 + 4 + 1;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int total = misc_off + 32;
  static constexpr int alloc = total + 1024;
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(q1_bytes % 1024 == 0 && q2_bytes % 1024 == 0 && k1_bytes % 1024 == 0 &&
                    k2_bytes % 1024 == 0,
                "operand tiles must stay 1024-byte aligned");
};

struct UnitQ {
  int bh, q0, nsteps;
  int kmask;  // key steps from kmask on need element masks
  int rot;    // iteration t visits key step (t + rot) mod nsteps
  // Key step of iteration t.  Every unit of a head would otherwise start at key
  // step 0 and all CTAs would reduce into the same dK rows at the same time;
  // the sums do not depend on the order.
  __device__ __forceinline__ int step(int t) const {
    int r = t + rot;
    if (r >= nsteps) r -= nsteps;
    return r;
  }
};

__device__ __forceinline__ UnitQ decode_unit(const BwdQtParams& p, int u) {
  const int nqt = (p.NQ + RQ - 1) / RQ;
  UnitQ w;
  w.bh = u / nqt;  // head-major: few heads active at once keeps K and dKacc in L2
  w.q0 = (nqt - 1 - u % nqt) * RQ;  // within a head, the query tiles that see most keys first
  const int off = p.NK - p.NQ;
  int nk = p.NK;  // keys [0, nk) are visible to some row of the tile
  int full = p.NK;  // keys [0, full) are visible to every row of the tile
  if (p.causal) {
    nk = min(p.NK, min(w.q0 + RQ - 1, p.NQ - 1) + off + 1);
    full = min(full, w.q0 + off + 1);
  }
  w.nsteps = (nk + CK - 1) / CK;
  w.kmask = full / CK;  // first step with a key some row cannot see (or past NK)
  const unsigned h = static_cast<unsigned>(u) * 2654435761u;
  w.rot = static_cast<int>((h >> 8) % static_cast<unsigned>(w.nsteps));
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

// This thread's query row, loaded once per unit:
//   b1 = -LSE1 log2e, b2 = -LSE2 log2e       (u_t = c_t S_t + b_t = log2 P_t)
//   gl = s1 dL ln2, gn = -s1 dL L             (s1 dS1 = P1 (gl (u1 - u2) + gn))
//   g2 = s2 dL                                (s2 dS2 = g2 (P2 - P1))
// Rows past NQ get zeros: their Q rows are zero-filled, so S = 0, P = 1 and
// every dS of theirs is 0.
struct RowRec {
  float b1, b2, gl, gn, g2;
};

// dS for one query row and KPW keys of a step (pairs of keys at a time, packed
// f32x2) into registers: w1/w2 receive the bf16 pairs of s1*dS1 and s2*dS2.
// MASK: key column c of this warpgroup is visible iff c <= last.
template <bool MASK, bool G1, bool G2>
__device__ __forceinline__ void form_ds_regs(const uint32_t (&s1)[KPW], const uint32_t (&s2)[KPW],
                                             const RowRec& rr, float c1, float c2, int last,
                                             uint32_t (&w1)[KPW / 2], uint32_t (&w2)[KPW / 2]) {
  const float2 C1 = make_float2(c1, c1), C2 = make_float2(c2, c2);
  const float2 B1 = make_float2(rr.b1, rr.b1), B2 = make_float2(rr.b2, rr.b2);
  const float2 GL = make_float2(rr.gl, rr.gl), GN = make_float2(rr.gn, rr.gn);
  const float2 G2v = make_float2(rr.g2, rr.g2);
  const float2 NEG1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int i = 0; i < KPW; i += 2) {
    const float2 S1 = make_float2(__uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
    const float2 S2 = make_float2(__uint_as_float(s2[i]), __uint_as_float(s2[i + 1]));
    const float2 u1 = __ffma2_rn(S1, C1, B1);
    const float2 u2 = __ffma2_rn(S2, C2, B2);
    const float2 P1 = make_float2(ex2(u1.x), ex2(u1.y));
    float2 d1 = make_float2(0.f, 0.f), d2 = make_float2(0.f, 0.f);
    if (G1) d1 = __fmul2_rn(P1, __ffma2_rn(__ffma2_rn(u2, NEG1, u1), GL, GN));
    if (G2) {
      const float2 P2 = make_float2(ex2(u2.x), ex2(u2.y));
      d2 = __fmul2_rn(__ffma2_rn(P1, NEG1, P2), G2v);
    }
    if (MASK) {
      const bool vx = i <= last, vy = i + 1 <= last;
      d1.x = vx ? d1.x : 0.f;
      d2.x = vx ? d2.x : 0.f;
      d1.y = vy ? d1.y : 0.f;
      d2.y = vy ? d2.y : 0.f;
    }
    if (G1) w1[i / 2] = pack_bf16(d1.x, d1.y);
    if (G2) w2[i / 2] = pack_bf16(d2.x, d2.y);
  }
}

template <bool G1, bool G2>
__device__ __forceinline__ void store_ds(const uint32_t (&w1)[KPW / 2],
                                         const uint32_t (&w2)[KPW / 2], int row, int c0,
                                         uint32_t ds1_row, uint32_t ds2_row) {
#pragma unroll
  for (int c = 0; c < KPW / 8; ++c) {
    const uint32_t sw = static_cast<uint32_t>(((c0 + c) ^ (row & 7)) << 4);
    if (G1) st_shared_v4(ds1_row + sw, w1[4 * c], w1[4 * c + 1], w1[4 * c + 2], w1[4 * c + 3]);
    if (G2) st_shared_v4(ds2_row + sw, w2[4 * c], w2[4 * c + 1], w2[4 * c + 2], w2[4 * c + 3]);
  }
}

// Adds 32 keys of one dK_t^T feature row into the fp32 accumulator: base
// points at the first key's row, feature f; rows are LDK floats apart.
template <int LDK, bool FULL>
__device__ __forceinline__ void red_dk(float* base, const uint32_t (&v)[32], int nvalid) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (FULL || i < nvalid) atomicAdd(base + i * LDK, __uint_as_float(v[i]));
}

template <int D1, int D2, int SEL>
__global__ void __launch_bounds__(NTHREADS, 1)
    streamkl_bwd_qt_kernel(const __grid_constant__ BwdQtParams p) {
  constexpr bool G1 = (SEL & 1) != 0, G2 = (SEL & 2) != 0;
  constexpr int NDT = (G1 ? 1 : 0) + (G2 ? 1 : 0);
  using Lay = QtLayout<D1, D2, NDT>;
  constexpr int KST = Lay::KSTAGES;
  constexpr int DSB = Lay::DSBUF;
  // dK accumulator row: the wanted sides only, teacher first
  constexpr int LDK = (G1 ? D1 : 0) + (G2 ? D2 : 0);
  constexpr int DK2_COL = G1 ? D1 : 0;
  // dQ accumulators from column 128: dQ1 then dQ2, or the one side asked for.
  // S buffers: one for both sides; two for one side, the second right after
  // that side's dQ (at most [256, 384), below dK1^T).
  constexpr uint32_t kColDQ2 = G1 ? kColDQ1 + D1 : kColDQ1;
  constexpr int NSB = (G1 && G2) ? 1 : 2;
  constexpr uint32_t kColSB1 = kColDQ1 + (G1 ? D1 : 0) + (G2 ? D2 : 0);
  static_assert(NSB == 1 || kColSB1 + 128 <= kColDK1, "TMEM budget exceeded");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* qfull = bars + 0;
  uint64_t* qempty = bars + 1;
  uint64_t* kfull = bars + 2;
  uint64_t* kempty = kfull + KST;
  uint64_t* sfull = kempty + KST;  // [2]
  uint64_t* sempty = sfull + 2;    // [2]
  // kempty[s] completes when the products of the step that used key stage s
  // are done: the producer may refill the stage, the dS buffer of that step is
  // free again and its dK^T is in TMEM.  One commit per step serves all three.
  uint64_t* dsfull = sempty + 2;
  uint64_t* dkempty = dsfull + DSB;  // [2]: dK1^T and dK2^T slots read out
  uint64_t* dqfull = dkempty + 2;
  uint64_t* dqempty = dqfull + 1;
  uint64_t* ufull = dqempty + 1;
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
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4 * NDS);  // every warp of every dS warpgroup
    }
    for (int s = 0; s < DSB; ++s) mbar_init(&dsfull[s], 4 * NDS);
    mbar_init(&dkempty[0], 4);
    mbar_init(&dkempty[1], 4);
    mbar_init(dqfull, 1);
    mbar_init(dqempty, 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ufull[s], 1);
      mbar_init(&uempty[s], 2 + 4 * NDS + 4);  // both UMMA issuers + dS warps + dK warps
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

  const int total = bwd_qt_units(p.BH, p.NQ);
  uint8_t* q1_s = smem + Lay::q1_off;
  uint8_t* q2_s = smem + Lay::q2_off;
  auto k1_s = [&](int s) { return smem + Lay::k_off + s * Lay::kstage_bytes; };
  auto k2_s = [&](int s) { return smem + Lay::k_off + s * Lay::kstage_bytes + Lay::k1_bytes; };
  auto ds1_s = [&](int b) { return smem + Lay::ds_off + b * NDT * Lay::ds_bytes; };
  auto ds2_s = [&](int b) {
    return smem + Lay::ds_off + b * NDT * Lay::ds_bytes + (G1 ? Lay::ds_bytes : 0);
  };
  const int off = p.NK - p.NQ;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int us = 0, ks = 0;
      uint32_t uph = 0, qph = 0, kph = 0;
      uint32_t armed_q = 0, armed_k[KST] = {};
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
        const UnitQ w = decode_unit(p, u);
        if (!(ok = mbar_wait(qempty, qph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(qfull, Lay::q1_bytes + Lay::q2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(q1_s + b * (RQ * 128), &p.tmQ1, qfull, b * 64, w.q0, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(q2_s + b * (RQ * 128), &p.tmQ2, qfull, b * 64, w.q0, w.bh);
        armed_q = qph + 1;
        qph ^= 1;
        for (int t = 0; t < w.nsteps; ++t) {
          const int k0 = w.step(t) * CK;
          if (!(ok = mbar_wait(&kempty[ks], kph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfull[ks], Lay::kstage_bytes);
#pragma unroll
          for (int b = 0; b < D1 / 64; ++b)
            tma_load_3d(k1_s(ks) + b * (CK * 128), &p.tmK1, &kfull[ks], b * 64, k0, w.bh);
#pragma unroll
          for (int b = 0; b < D2 / 64; ++b)
            tma_load_3d(k2_s(ks) + b * (CK * 128), &p.tmK2, &kfull[ks], b * 64, k0, w.bh);
          armed_k[ks] = kph + 1;
          if (++ks == KST) {
            ks = 0;
            kph ^= 1;
          }
        }
        if (!ok) break;
        next = static_cast<int>(gridDim.x) + atomicAdd(p.counter, 1);
      }
      if (!ok) {
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        if (armed_q) mbar_wait(qfull, armed_q - 1, dctl);
        for (int s = 0; s < KST; ++s)
          if (armed_k[s]) mbar_wait(&kfull[s], armed_k[s] - 1, dctl);
      }
    }
  } else if (warp == 1 || warp == S_WARP) {
    // ------------------------------------------------------------ UMMA issuers
    // Two threads feed the tensor pipe: the S products come from warp S_WARP,
    // the contractions from warp 1.  The queue in front of the pipe holds about
    // one product, so a single issuing thread leaves the pipe idle whenever it
    // checks a barrier or waits; with two, one stream's waits are filled by the
    // other's products.  A commit tracks the issuing thread's own products,
    // which is what each barrier below means: sfull the S of a step, kempty the
    // contractions of a step (whose dS implies that step's S was done).
    if (lane == 0) {
      const bool s_role = warp == S_WARP;
      constexpr uint32_t idS = idesc_bf16(RQ, CK);           // S: M=128 queries, N=64 keys
      constexpr uint32_t idQ1 = idesc_bf16(RQ, D1, 0, 1);    // dQ1: B = K1 MN-major
      constexpr uint32_t idQ2 = idesc_bf16(RQ, D2, 0, 1);
      constexpr uint32_t idK1 = idesc_bf16(D1, CK, 1, 1);    // dK1^T: A = Q1 MN-major
      constexpr uint32_t idK2 = idesc_bf16(D2, CK, 1, 1);
      const uint32_t q1a = smem_u32(q1_s), q2a = smem_u32(q2_s);
      const uint64_t q1d = sdesc_sw128(q1a, 16, 1024), q2d = sdesc_sw128(q2a, 16, 1024);
      // Q tiles read MN-major for dK^T: 64-feature chunks 16 KB apart
      const uint64_t q1m = sdesc_sw128(q1a, RQ * 128, 1024), q2m = sdesc_sw128(q2a, RQ * 128, 1024);
      int us = 0, ks_s = 0, ks_r = 0, db = 0, sb = 0;
      uint32_t uph = 0, qph = 0, kph_s = 0, dqph = 0;
      uint32_t sph = 0;  // bit b: parity of S buffer b's current use
      uint32_t dkph[2] = {0, 0};
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
        const UnitQ w = decode_unit(p, u);
        if (s_role) {
          if (!(ok = mbar_wait(qfull, qph, ctl))) break;
          qph ^= 1;
          for (int t = 0; t < w.nsteps; ++t) {
            if (!(ok = mbar_wait(&kfull[ks_s], kph_s, ctl))) break;
            if (!(ok = mbar_wait(&sempty[sb], ((sph >> sb) & 1u) ^ 1u, ctl))) break;
            tc_fence_after();
            const uint32_t scol = tmem_base + (sb == 0 ? 0u : kColSB1);
            const uint64_t k1d = sdesc_sw128(smem_u32(k1_s(ks_s)), 16, 1024);
            const uint64_t k2d = sdesc_sw128(smem_u32(k2_s(ks_s)), 16, 1024);
#pragma unroll
            for (int kk = 0; kk < D1 / 16; ++kk) {
              const uint32_t o = (kk & 3) * 32;
              umma_bf16_ss(scol + kColS1, sdesc_advance(q1d, (kk >> 2) * (RQ * 128) + o),
                           sdesc_advance(k1d, (kk >> 2) * (CK * 128) + o), idS, kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < D2 / 16; ++kk) {
              const uint32_t o = (kk & 3) * 32;
              umma_bf16_ss(scol + kColS2, sdesc_advance(q2d, (kk >> 2) * (RQ * 128) + o),
                           sdesc_advance(k2d, (kk >> 2) * (CK * 128) + o), idS, kk > 0);
            }
            umma_commit(&sfull[sb]);
            sph ^= 1u << sb;
            if (NSB == 2) sb ^= 1;
            if (++ks_s == KST) {
              ks_s = 0;
              kph_s ^= 1;
            }
          }
          if (!ok) break;
          continue;
        }
        for (int t = 0; t < w.nsteps; ++t) {
          if (!(ok = mbar_wait(&dsfull[db], dsph[db], ctl))) break;
          dsph[db] ^= 1;
          if (t == 0) {  // the previous unit's dQ has been read out of TMEM
            if (!(ok = mbar_wait(dqempty, dqph ^ 1, ctl))) break;
            dqph ^= 1;
          }
          tc_fence_after();
          // Descriptors of this step's operands are built once; each UMMA below
          // adds a constant offset.
          const uint32_t ds1a = smem_u32(ds1_s(db)), ds2a = smem_u32(ds2_s(db));
          const uint64_t d1k = sdesc_sw128(ds1a, 16, 1024), d2k = sdesc_sw128(ds2a, 16, 1024);
          const uint64_t d1m = sdesc_sw128(ds1a, CK * 128, 1024), d2m = sdesc_sw128(ds2a, CK * 128, 1024);
          const uint64_t k1m = sdesc_sw128(smem_u32(k1_s(ks_r)), CK * 128, 1024);
          const uint64_t k2m = sdesc_sw128(smem_u32(k2_s(ks_r)), CK * 128, 1024);
          const uint32_t acc0 = t > 0;
          // dQ_t += (s_t dS_t) K_t : A = dS (K-major, 128B rows of 64 keys), B = K_t
          // read MN-major (features contiguous; 64-feature chunks 8 KB apart).
          if (G1 && p.want_dq1) {
#pragma unroll
            for (int kk = 0; kk < CK / 16; ++kk)
              umma_bf16_ss(tmem_base + kColDQ1, sdesc_advance(d1k, kk * 32),
                           sdesc_advance(k1m, kk * 2048), idQ1, kk > 0 ? 1u : acc0);
          }
          if (G2 && p.want_dq2) {
#pragma unroll
            for (int kk = 0; kk < CK / 16; ++kk)
              umma_bf16_ss(tmem_base + kColDQ2, sdesc_advance(d2k, kk * 32),
                           sdesc_advance(k2m, kk * 2048), idQ2, kk > 0 ? 1u : acc0);
          }
          // dK_t^T = Q_t^T (s_t dS_t) : A = Q tile read MN-major (64-feature chunks
          // 16 KB apart), B = dS read MN-major (64 keys contiguous per query).
          if (G1) {
            if (!(ok = mbar_wait(&dkempty[0], dkph[0] ^ 1, ctl))) break;
            dkph[0] ^= 1;
            tc_fence_after();
            if (p.want_dk1) {
#pragma unroll
              for (int kk = 0; kk < RQ / 16; ++kk)
                umma_bf16_ss(tmem_base + kColDK1, sdesc_advance(q1m, kk * 2048),
                             sdesc_advance(d1m, kk * 2048), idK1, kk > 0);
            }
          }
          if (G2) {
            if (!(ok = mbar_wait(&dkempty[1], dkph[1] ^ 1, ctl))) break;
            dkph[1] ^= 1;
            tc_fence_after();
            if (p.want_dk2) {
#pragma unroll
              for (int kk = 0; kk < RQ / 16; ++kk)
                umma_bf16_ss(tmem_base + kColDK2, sdesc_advance(q2m, kk * 2048),
                             sdesc_advance(d2m, kk * 2048), idK2, kk > 0);
            }
          }
          umma_commit(&kempty[ks_r]);  // step done: K stage free, dS buffer free, dK^T ready
          if (++db == DSB) db = 0;
          if (++ks_r == KST) ks_r = 0;
        }
        if (!ok) break;
        umma_commit(dqfull);
        umma_commit(qempty);
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
  } else if (warp < DK_WARP0) {
    // ------------------------------------------------------------ dS warpgroups
    const int part = (warp - 2) >> 2;  // keys [part*KPW, part*KPW + KPW) of each step
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int us = 0, db = 0, sb = 0;
    uint32_t uph = 0;
    uint32_t sph = 0;  // bit b: parity of S buffer b's current use
    int pks = -1;        // K stage of the previous step (-1: none yet)
    uint32_t pkph = 0;   // its phase
    int cks = 0;         // K stage of the current step
    uint32_t ckph = 0;
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
      const UnitQ w = decode_unit(p, u);
      const int i = w.q0 + r;
      RowRec rr{0.f, 0.f, 0.f, 0.f, 0.f};
      if (i < p.NQ) {
        const size_t o = static_cast<size_t>(w.bh) * p.NQ + i;
        const float g = __ldg(p.dL + o);
        rr.b1 = -__ldg(p.LSE1 + o) * kLog2e;
        rr.b2 = -__ldg(p.LSE2 + o) * kLog2e;
        rr.gl = p.s1 * g * kLn2;
        rr.gn = -p.s1 * g * __ldg(p.L + o);
        rr.g2 = p.s2 * g;
      }
      // last key column this row sees, counted from this warpgroup's first key
      const int lim = (p.causal ? min(p.NK - 1, i + off) : p.NK - 1) - part * KPW;
      const uint32_t rowoff = static_cast<uint32_t>(r) * 128;
      for (int t = 0; t < w.nsteps; ++t) {
        const int ks = w.step(t);
        const int k0 = ks * CK;
        if (!(ok = mbar_wait(&sfull[sb], (sph >> sb) & 1u, ctl))) break;
        sph ^= 1u << sb;
        tc_fence_after();
        const uint32_t scol = tl + (sb == 0 ? 0u : kColSB1);
        uint32_t a[KPW], b[KPW];
        tmem_ld_32x32b<KPW>(scol + kColS1 + part * KPW, a);
        tmem_ld_32x32b<KPW>(scol + kColS2 + part * KPW, b);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sempty[sb]);
        if (NSB == 2) sb ^= 1;
        const bool masked = ks >= w.kmask;
        const int last = lim - k0;
        const uint32_t r1 = smem_u32(ds1_s(db)) + rowoff, r2 = smem_u32(ds2_s(db)) + rowoff;
        // dS is formed in registers first, with the whole segment's arithmetic
        // in flight at once, while the previous step's contractions may still
        // read the buffer; it is stored once they are done (the previous
        // step's key stage released).
        uint32_t w1[KPW / 2], w2[KPW / 2];
        if (masked)
          form_ds_regs<true, G1, G2>(a, b, rr, p.c1, p.c2, last, w1, w2);
        else
          form_ds_regs<false, G1, G2>(a, b, rr, p.c1, p.c2, 0, w1, w2);
        if (pks >= 0 && !(ok = mbar_wait(&kempty[pks], pkph, ctl))) break;
        store_ds<G1, G2>(w1, w2, r, part * (KPW / 8), r1, r2);
        pks = cks;
        pkph = ckph;
        if (++cks == KST) {
          cks = 0;
          ckph ^= 1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dsfull[db]);
        if (++db == DSB) db = 0;
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ dK / dQ warpgroup
    const int quarter = warp & 3;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    // dK_t^T rows are features: M = 128 puts feature f in lane f; M = 64 puts
    // features 16q..16q+15 in lanes 32q..32q+15.
    const int f1 = (D1 == 128) ? quarter * 32 + lane : (lane < 16 ? quarter * 16 + lane : -1);
    const int f2 = (D2 == 128) ? quarter * 32 + lane : (lane < 16 ? quarter * 16 + lane : -1);
    int us = 0;
    uint32_t uph = 0, dqph = 0;
    int cks = 0;
    uint32_t ckph = 0;
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
      const UnitQ w = decode_unit(p, u);
      for (int t = 0; t < w.nsteps; ++t) {
        const int k0 = w.step(t) * CK;
        if (!(ok = mbar_wait(&kempty[cks], ckph, ctl))) break;
        if (++cks == KST) {
          cks = 0;
          ckph ^= 1;
        }
        tc_fence_after();
        const int nvalid = min(CK, p.NK - k0);
        float* base = p.dKacc + (static_cast<size_t>(w.bh) * p.NK + k0) * LDK;
#pragma unroll
        for (int tsel = 0; tsel < 2; ++tsel) {
          if ((tsel == 0 && !G1) || (tsel == 1 && !G2)) continue;
          const bool want = tsel == 0 ? p.want_dk1 : p.want_dk2;
          const int f = tsel == 0 ? f1 : DK2_COL + f2;
          const bool fok = (tsel == 0 ? f1 : f2) >= 0;
          const uint32_t col = tl + (tsel == 0 ? kColDK1 : kColDK2);
          // both halves of 32 keys into registers, the slot released, then the reductions
          uint32_t v0[32], v1[32];
          if (want) {
            tmem_ld_32x32b_x32(col, v0);
            tmem_ld_32x32b_x32(col + 32, v1);
            tmem_ld_wait();
            reg_fence(v0);
            reg_fence(v1);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dkempty[tsel]);
          if (want && fok) {
            if (nvalid == CK)
              red_dk<LDK, true>(base + f, v0, 32);
            else
              red_dk<LDK, false>(base + f, v0, nvalid);
          }
          if (want && fok) {
            if (nvalid == CK)
              red_dk<LDK, true>(base + 32 * LDK + f, v1, 32);
            else
              red_dk<LDK, false>(base + 32 * LDK + f, v1, nvalid - 32);
          }
        }
      }
      if (!ok) break;
      // Unit epilogue: dQ accumulators (thread = query row) to bf16.
      if (!(ok = mbar_wait(dqfull, dqph, ctl))) break;
      dqph ^= 1;
      tc_fence_after();
      const int i = w.q0 + quarter * 32 + lane;
      const bool row_ok = i < p.NQ;
#pragma unroll
      for (int tsel = 0; tsel < 2; ++tsel) {
        if ((tsel == 0 && !G1) || (tsel == 1 && !G2)) continue;
        const bool want = tsel == 0 ? p.want_dq1 : p.want_dq2;
        if (!want) continue;
        constexpr int DMAX = D1 > D2 ? D1 : D2;
        const int D = tsel == 0 ? D1 : D2;
        __nv_bfloat16* dst =
            (tsel == 0 ? p.dQ1 : p.dQ2) + (static_cast<size_t>(w.bh) * p.NQ + i) * D;
        const uint32_t col0 = tl + (tsel == 0 ? kColDQ1 : kColDQ2);
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
      if (lane == 0) mbar_arrive(dqempty);
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

template <int D1, int D2, int SEL>
cudaError_t launch_t(const BwdQtParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = QtLayout<D1, D2, (SEL == 3) ? 2 : 1>::alloc;
  auto kern = streamkl_bwd_qt_kernel<D1, D2, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int SEL>
cudaError_t launch_sel(const BwdQtParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128, SEL>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64, SEL>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_bwd_qt(const BwdQtParams& p, int d1, int d2, int sel, int grid,
                          cudaStream_t stream) {
  if (sel == 1) return launch_sel<1>(p, d1, d2, grid, stream);
  if (sel == 2) return launch_sel<2>(p, d1, d2, grid, stream);
  if (sel == 3) return launch_sel<3>(p, d1, d2, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace skl
