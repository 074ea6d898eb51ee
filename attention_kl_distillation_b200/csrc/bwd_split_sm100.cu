// bwd_split_sm100.cu -- the backward as two separate passes, for sm_100a.
//
// StreamKL summary page, "Metodologia" section 2 ("Fusione del Kernel"): the
// fused backward accumulates dQ with atomics while that buffer fits in L2 and
// switches to separate kernels when contention grows; the ablation compares
// the two ("Risultati Sperimentali").  This file is the separate variant: one
// kernel template run twice,
//
//   dK pass  resident 128-key tile R = K, streamed 64-query tiles C = Q:
//            S^T = K Q^T,  dK_t += (s_t dS_t)^T Q_t
//   dQ pass  resident 128-query tile R = Q, streamed 64-key tiles C = K:
//            S = Q K^T,    dQ_t += (s_t dS_t) K_t
//
// Both have the same shape, OUT += dS . C with dS = f(R C^T): S (M=128, N=64)
// comes from a UMMA with both operands in shared memory, dS is written in bf16
// to TMEM by the compute warps and the product is a UMMA whose A operand is
// that TMEM tile.  S of successive steps alternates between two TMEM slots and
// dS is written into the slot it came from, so S of step t+1 is computed while
// dS of step t is formed and contracted.  Each pass regenerates P1, P2 from the saved LSEs and keeps
// its gradient in TMEM for the whole unit, so no accumulator in global memory
// and no atomics are needed; the price is recomputing S and the exponentials
// once more than the fused kernel does.
//
// Roles: warp 0 TMA producer (R once per unit, C tiles into a ring, and for the
// dK pass the per-query records of each step) and unit dispenser; warp 1 TMEM
// owner and UMMA issuer; warps 2..17 four compute warpgroups, each owning 16 of
// the 64 streamed rows of a step (thread = resident row = TMEM lane).
// TMEM: two slots of 128 columns at 0 and 128, each S1 [0,64) S2 [64,128) of
//       one step; OUT1 [256, 256+d1) OUT2 [256+d1, 256+d1+d2).  A compute
//       warpgroup that owns streamed rows [16p, 16p+16) reads S1 columns
//       [16p, 16p+16) of the slot and writes its bf16 dS1 and dS2 over them
//       ([16p, 16p+8) and [16p+8, 16p+16)): columns only it has read, and the
//       eight columns one K16 step of the product reads as its A operand.
#include "kernels.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

namespace skl {
namespace {

constexpr int RB = 128;                     // resident rows per unit (UMMA M)
constexpr int CB = 64;                      // streamed rows per step
constexpr int NDS = 4;                      // compute warpgroups
constexpr int CPW = CB / NDS;               // streamed rows per compute warpgroup
constexpr int NTHREADS = (2 + 4 * NDS) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr uint32_t kSlotCols = 128, kColS2 = 64, kColOut = 256;
constexpr int kNegInf = -(1 << 30), kPosInf = (1 << 30);

template <BwdPass PASS, int D1, int D2>
struct SplitLayout {
  static constexpr int r1_bytes = RB * D1 * 2;
  static constexpr int r2_bytes = RB * D2 * 2;
  static constexpr int c1_bytes = CB * D1 * 2;
  static constexpr int c2_bytes = CB * D2 * 2;
  static constexpr int rr_bytes = PASS == BwdPass::kDK ? CB * kRowRec * 4 : 0;
  static constexpr int stage_bytes = c1_bytes + c2_bytes + rr_bytes;
  static constexpr int r_off = 0;
  static constexpr int c_off = r1_bytes + r2_bytes;
  static constexpr int nst_fit = (232448 - 1024 - 512 - c_off) / stage_bytes;
  static constexpr int NST = nst_fit > 6 ? 6 : nst_fit;
  static constexpr int bar_off = c_off + NST * stage_bytes;
  // rfull rempty cfull[NST] cempty[NST] sfull[2] dsfull[2] ofull oempty ufull[2] uempty[2] drain
  static constexpr int nbar = 2 + 2 * NST + 4 + 2 + 4 + 1;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int alloc = misc_off + 32 + 1024;
  static_assert(NST >= 3, "streamed ring too shallow");
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(r1_bytes % 1024 == 0 && r2_bytes % 1024 == 0 && c1_bytes % 1024 == 0 &&
                    c2_bytes % 1024 == 0 && stage_bytes % 1024 == 0,
                "operand tiles must stay 1024-byte aligned");
};

// One work unit: a resident tile of 128 rows of head bh and the streamed tiles
// it meets, visited from a unit-dependent rotation (sums do not depend on order).
struct UnitS {
  int bh, r0, c_first, nsteps, rot;
  __device__ __forceinline__ int c0(int t) const {
    int r = t + rot;
    if (r >= nsteps) r -= nsteps;
    return (c_first + r) * CB;
  }
};

template <BwdPass PASS>
__device__ __forceinline__ UnitS decode_split(const BwdSplitParams& p, int u) {
  UnitS w;
  const int off = p.NK - p.NQ;
  if (PASS == BwdPass::kDK) {
    const int nrt = (p.NK + RB - 1) / RB;
    w.bh = u / nrt;
    const int rt = u % nrt;  // key tiles with the most visible queries first
    w.r0 = rt * RB;
    int first = 0;
    if (p.causal) {
      const int q = w.r0 - off;  // first query row that sees key r0
      first = q > 0 ? q / CB : 0;
    }
    w.c_first = first;
    w.nsteps = p.NQpad / CB - first;
    w.rot = static_cast<int>((static_cast<unsigned>(rt) * 2654435761u) %
                             static_cast<unsigned>(w.nsteps));
  } else {
    const int nrt = (p.NQ + RB - 1) / RB;
    w.bh = u / nrt;
    const int rt = nrt - 1 - u % nrt;  // query tiles that see the most keys first
    w.r0 = rt * RB;
    const int nct = (p.NK + CB - 1) / CB;
    int last = nct;
    if (p.causal) last = min(nct, (min(w.r0 + RB - 1, p.NQ - 1) + off) / CB + 1);
    w.c_first = 0;
    w.nsteps = last;
    w.rot = static_cast<int>((static_cast<unsigned>(rt) * 2654435761u) %
                             static_cast<unsigned>(w.nsteps));
  }
  return w;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// dS for one resident row and CPW streamed rows (pairs at a time, packed
// f32x2).  Per streamed element the record fields are nb1 = -LSE1 log2e,
// nb2 = -LSE2 log2e, nL = -L, g1 = s1 dL, g2 = s2 dL of the query involved:
//   u_t = c_t S_t + nb_t = log2 P_t
//   dS1 = g1 P1 (ln2 (u1 - u2) - L),   dS2 = g2 (P2 - P1)
// Visible streamed rows i satisfy lo <= i <= hi (MASK only).
// Records come from shared memory per column (dK pass, COLREC) or are the
// same for every column (dQ pass: the thread's own query row).  G1/G2: which
// of dS1, dS2 the pass contracts; only those are formed, and without dS2 the
// student's exponential is not taken (dS1 needs the student only through u2).
template <bool MASK, bool COLREC, bool G1, bool G2>
__device__ __forceinline__ void form_ds(const uint32_t (&s1)[CPW], const uint32_t (&s2)[CPW],
                                        const float* rr, const float (&rec)[5], float c1,
                                        float c2, int lo, int hi, uint32_t (&w1)[CPW / 2],
                                        uint32_t (&w2)[CPW / 2]) {
  const float2 C1 = make_float2(c1, c1), C2 = make_float2(c2, c2);
  const float2 NEG1 = make_float2(-1.f, -1.f), LN2 = make_float2(kLn2, kLn2);
#pragma unroll
  for (int q = 0; q < CPW; q += 4) {
    float4 nb1, nb2, nL, g1, g2;
    if (COLREC) {
      nb1 = ld_shared_f4(rr + 0 * CB + q);
      nb2 = ld_shared_f4(rr + 1 * CB + q);
      nL = G1 ? ld_shared_f4(rr + 2 * CB + q) : float4{};
      g1 = G1 ? ld_shared_f4(rr + 3 * CB + q) : float4{};
      g2 = G2 ? ld_shared_f4(rr + 4 * CB + q) : float4{};
    } else {
      nb1 = make_float4(rec[0], rec[0], rec[0], rec[0]);
      nb2 = make_float4(rec[1], rec[1], rec[1], rec[1]);
      nL = make_float4(rec[2], rec[2], rec[2], rec[2]);
      g1 = make_float4(rec[3], rec[3], rec[3], rec[3]);
      g2 = make_float4(rec[4], rec[4], rec[4], rec[4]);
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
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
        const bool vx = i >= lo && i <= hi, vy = i + 1 >= lo && i + 1 <= hi;
        d1.x = vx ? d1.x : 0.f;
        d2.x = vx ? d2.x : 0.f;
        d1.y = vy ? d1.y : 0.f;
        d2.y = vy ? d2.y : 0.f;
      }
      if (G1) w1[q / 2 + e] = pack_bf16(d1.x, d1.y);
      if (G2) w2[q / 2 + e] = pack_bf16(d2.x, d2.y);
    }
  }
}

template <BwdPass PASS, int D1, int D2, int SEL>
__global__ void __launch_bounds__(NTHREADS, 1)
    streamkl_bwd_split_kernel(const __grid_constant__ BwdSplitParams p) {
  // SEL: the gradient sides this pass writes (1 teacher: out1, 2 student: out2,
  // 3 both); a one-sided instance forms, stores and contracts that side's dS only.
  constexpr bool G1 = (SEL & 1) != 0, G2 = (SEL & 2) != 0;
  using Lay = SplitLayout<PASS, D1, D2>;
  constexpr int NST = Lay::NST;
  constexpr bool DK = PASS == BwdPass::kDK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* rfull = bars + 0;
  uint64_t* rempty = bars + 1;
  uint64_t* cfull = bars + 2;
  uint64_t* cempty = cfull + NST;
  uint64_t* sfull = cempty + NST;  // [2]: S of a step is in the slot
  uint64_t* dsfull = sfull + 2;    // [2]: dS of a step has replaced it
  uint64_t* ofull = dsfull + 2;
  uint64_t* oempty = ofull + 1;
  uint64_t* ufull = oempty + 1;  // [2]
  uint64_t* uempty = ufull + 2;  // [2]
  uint64_t* drain = uempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 4);
  volatile int* unit_slot = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 8);  // [2]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(rfull, 1);
    mbar_init(rempty, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&dsfull[s], 4 * NDS);
      mbar_init(&ufull[s], 1);
      mbar_init(&uempty[s], 1 + 4 * NDS);  // MMA thread + compute warps
    }
    mbar_init(ofull, 1);
    mbar_init(oempty, 4 * NDS);
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmR1);
    tma_prefetch_desc(&p.tmR2);
    tma_prefetch_desc(&p.tmC1);
    tma_prefetch_desc(&p.tmC2);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int total =
      p.BH * (DK ? (p.NK + RB - 1) / RB : (p.NQ + RB - 1) / RB);
  uint8_t* r1_s = smem + Lay::r_off;
  uint8_t* r2_s = smem + Lay::r_off + Lay::r1_bytes;
  auto c1_s = [&](int s) { return smem + Lay::c_off + s * Lay::stage_bytes; };
  auto c2_s = [&](int s) { return smem + Lay::c_off + s * Lay::stage_bytes + Lay::c1_bytes; };
  auto rr_s = [&](int s) {
    return reinterpret_cast<float*>(smem + Lay::c_off + s * Lay::stage_bytes + Lay::c1_bytes +
                                    Lay::c2_bytes);
  };
  const int off = p.NK - p.NQ;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int us = 0, cs = 0;
      uint32_t uph = 0, rph = 0, cph = 0;
      uint32_t armed_r = 0, armed_c[NST] = {};
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
        const UnitS w = decode_split<PASS>(p, u);
        if (!(ok = mbar_wait(rempty, rph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(rfull, Lay::r1_bytes + Lay::r2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(r1_s + b * (RB * 128), &p.tmR1, rfull, b * 64, w.r0, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(r2_s + b * (RB * 128), &p.tmR2, rfull, b * 64, w.r0, w.bh);
        armed_r = rph + 1;
        rph ^= 1;
        for (int t = 0; t < w.nsteps; ++t) {
          const int c0 = w.c0(t);
          if (!(ok = mbar_wait(&cempty[cs], cph ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&cfull[cs], Lay::stage_bytes);
#pragma unroll
          for (int b = 0; b < D1 / 64; ++b)
            tma_load_3d(c1_s(cs) + b * (CB * 128), &p.tmC1, &cfull[cs], b * 64, c0, w.bh);
#pragma unroll
          for (int b = 0; b < D2 / 64; ++b)
            tma_load_3d(c2_s(cs) + b * (CB * 128), &p.tmC2, &cfull[cs], b * 64, c0, w.bh);
          if (DK)
            bulk_load(rr_s(cs), p.rowrec + (static_cast<size_t>(w.bh) * p.NQpad + c0) * kRowRec,
                      Lay::rr_bytes, &cfull[cs]);
          armed_c[cs] = cph + 1;
          if (++cs == NST) {
            cs = 0;
            cph ^= 1;
          }
        }
        if (!ok) break;
        next = static_cast<int>(gridDim.x) + atomicAdd(p.counter, 1);
      }
      if (!ok) {
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        if (armed_r) mbar_wait(rfull, armed_r - 1, dctl);
        for (int s = 0; s < NST; ++s)
          if (armed_c[s]) mbar_wait(&cfull[s], armed_c[s] - 1, dctl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(RB, CB);         // S: M=128 resident, N=64 streamed
      constexpr uint32_t idO1 = idesc_bf16(RB, D1, 0, 1);  // OUT1: A = dS (TMEM), B = C1 MN-major
      constexpr uint32_t idO2 = idesc_bf16(RB, D2, 0, 1);
      const uint64_t r1d = sdesc_sw128(smem_u32(r1_s), 16, 1024);
      const uint64_t r2d = sdesc_sw128(smem_u32(r2_s), 16, 1024);
      // slot_s: the slot the next S goes to; slot_r: the slot of the step whose
      // product is next.  A slot's S is issued only after the product that read
      // its previous dS (UMMAs of this thread execute in issue order).
      int us = 0, cs_s = 0, cs_r = 0, slot_s = 0, slot_r = 0;
      uint32_t uph = 0, rph = 0, cph_s = 0, oph = 0;
      uint32_t dsph = 0;  // bit s: parity of slot s's dsfull
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
        const UnitS w = decode_split<PASS>(p, u);
        if (!(ok = mbar_wait(rfull, rph, ctl))) break;
        rph ^= 1;
        auto issue_s = [&]() -> bool {
          if (!mbar_wait(&cfull[cs_s], cph_s, ctl)) return false;
          tc_fence_after();
          const uint32_t sd = tmem_base + slot_s * kSlotCols;
          const uint64_t c1d = sdesc_sw128(smem_u32(c1_s(cs_s)), 16, 1024);
          const uint64_t c2d = sdesc_sw128(smem_u32(c2_s(cs_s)), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D1 / 16; ++kk) {
            const uint32_t o = (kk & 3) * 32;
            umma_bf16_ss(sd, sdesc_advance(r1d, (kk >> 2) * (RB * 128) + o),
                         sdesc_advance(c1d, (kk >> 2) * (CB * 128) + o), idS, kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D2 / 16; ++kk) {
            const uint32_t o = (kk & 3) * 32;
            umma_bf16_ss(sd + kColS2, sdesc_advance(r2d, (kk >> 2) * (RB * 128) + o),
                         sdesc_advance(c2d, (kk >> 2) * (CB * 128) + o), idS, kk > 0);
          }
          umma_commit(&sfull[slot_s]);
          slot_s ^= 1;
          if (++cs_s == NST) {
            cs_s = 0;
            cph_s ^= 1;
          }
          return true;
        };
        if (!(ok = issue_s())) break;
        for (int t = 0; t < w.nsteps && ok; ++t) {
          if (t + 1 < w.nsteps && !(ok = issue_s())) break;
          if (!(ok = mbar_wait(&dsfull[slot_r], (dsph >> slot_r) & 1u, ctl))) break;
          dsph ^= 1u << slot_r;
          if (t == 0) {
            if (!(ok = mbar_wait(oempty, oph ^ 1, ctl))) break;
            oph ^= 1;
          }
          tc_fence_after();
          // C tiles read MN-major: features contiguous, 64-feature chunks 8 KB apart
          const uint64_t c1m = sdesc_sw128(smem_u32(c1_s(cs_r)), CB * 128, 1024);
          const uint64_t c2m = sdesc_sw128(smem_u32(c2_s(cs_r)), CB * 128, 1024);
          const uint32_t dsa = tmem_base + slot_r * kSlotCols;
          // OUT_t += dS_t (TMEM; K16 step kk: dS1 in columns [16kk, 16kk+8), dS2 in
          // [16kk+8, 16kk+16) of the slot) . C_t (read MN-major: features
          // contiguous, 64-feature chunks 8 KB apart).
#pragma unroll
          for (int kk = 0; kk < CB / 16; ++kk) {
            if (G1)
              umma_bf16_ts(tmem_base + kColOut, dsa + kk * 16, sdesc_advance(c1m, kk * 2048), idO1,
                           (t > 0 || kk > 0));
            if (G2)
              umma_bf16_ts(tmem_base + kColOut + D1, dsa + kk * 16 + 8, sdesc_advance(c2m, kk * 2048),
                           idO2, (t > 0 || kk > 0));
          }
          umma_commit(&cempty[cs_r]);
          slot_r ^= 1;
          if (++cs_r == NST) cs_r = 0;
        }
        if (!ok) break;
        umma_commit(ofull);
        umma_commit(rempty);
      }
      umma_commit(drain);
      volatile int zero = 0;
      WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
      mbar_wait(drain, 0, dctl);
    }
  } else {
    // ------------------------------------------------------------ compute warpgroups
    const int part = (warp - 2) >> 2;  // streamed rows [part*CPW, part*CPW + CPW) of each step
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // resident row within the tile (TMEM lane)
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    int us = 0, cs = 0, slot = 0;
    uint32_t uph = 0, cph = 0, oph = 0;
    uint32_t sph = 0;  // bit s: parity of slot s's sfull
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
      const UnitS w = decode_split<PASS>(p, u);
      const int row = w.r0 + j;  // key (dK pass) or query (dQ pass)
      float rec[5] = {0.f, 0.f, 0.f, 0.f, 0.f};
      if (!DK && row < p.NQ) {
        const float* r = p.rowrec + (static_cast<size_t>(w.bh) * p.NQpad + (row / CB) * CB) *
                                        kRowRec + (row % CB);
#pragma unroll
        for (int f = 0; f < 5; ++f) rec[f] = r[f * CB];
      }
      for (int t = 0; t < w.nsteps; ++t) {
        const int cc = w.c0(t) + part * CPW;  // first streamed row of this warpgroup
        if (DK) {
          if (!(ok = mbar_wait(&cfull[cs], cph, ctl))) break;  // per-query records of the step
        }
        if (!(ok = mbar_wait(&sfull[slot], (sph >> slot) & 1u, ctl))) break;
        sph ^= 1u << slot;
        tc_fence_after();
        const uint32_t scol = tl + slot * kSlotCols + part * CPW;
        uint32_t a[CPW], b[CPW];
        tmem_ld_32x32b_x16(scol, a);
        tmem_ld_32x32b_x16(scol + kColS2, b);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        const int c0 = w.c0(t);
        bool masked;
        int lo = kNegInf, hi = kPosInf;
        if (DK) {  // resident key `row`, streamed queries cc + i
          masked = (p.causal && c0 + off < w.r0 + RB - 1) || (w.r0 + RB > p.NK);
          if (row >= p.NK) lo = kPosInf;
          else if (p.causal) lo = row - off - cc;
        } else {  // resident query `row`, streamed keys cc + i
          masked = (p.causal && c0 + CB - 1 > w.r0 + off) || (c0 + CB > p.NK);
          hi = p.NK - 1 - cc;
          if (p.causal) hi = min(hi, row + off - cc);
        }
        uint32_t w1[CPW / 2], w2[CPW / 2];
        const float* rr = DK ? rr_s(cs) + part * CPW : nullptr;
        if (masked)
          form_ds<true, DK, G1, G2>(a, b, rr, rec, p.c1, p.c2, lo, hi, w1, w2);
        else
          form_ds<false, DK, G1, G2>(a, b, rr, rec, p.c1, p.c2, lo, hi, w1, w2);
        // dS over this warpgroup's own S1 columns of the slot
        if (G1) tmem_st_32x32b_x8(scol, w1);
        if (G2) tmem_st_32x32b_x8(scol + CPW / 2, w2);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dsfull[slot]);
        slot ^= 1;
        if (++cs == NST) {
          cs = 0;
          cph ^= 1;
        }
      }
      if (!ok) break;
      // Unit epilogue: this warpgroup converts its quarter of the OUT columns.
      if (!(ok = mbar_wait(ofull, oph, ctl))) break;
      oph ^= 1;
      tc_fence_after();
      const bool row_ok = row < (DK ? p.NK : p.NQ);
      const size_t nrows = DK ? p.NK : p.NQ;
#pragma unroll
      for (int tsel = 0; tsel < 2; ++tsel) {
        if ((tsel == 0 && !G1) || (tsel == 1 && !G2)) continue;
        __nv_bfloat16* dst = tsel == 0 ? p.out1 : p.out2;
        constexpr int DW1 = D1 / NDS, DW2 = D2 / NDS;  // columns per warpgroup
        const int D = tsel == 0 ? D1 : D2;
        const int DW = tsel == 0 ? DW1 : DW2;
        if (!dst) continue;
        const uint32_t col = tl + kColOut + (tsel == 0 ? 0 : D1) + part * DW;
        __nv_bfloat16* drow = dst + (static_cast<size_t>(w.bh) * nrows + row) * D + part * DW;
#pragma unroll
        for (int c = 0; c < (DW1 > DW2 ? DW1 : DW2); c += 16) {
          if (c >= DW) break;
          uint32_t v[16];
          tmem_ld_32x32b_x16(col + c, v);
          tmem_ld_wait();
          reg_fence(v);
          if (row_ok) {
#pragma unroll
            for (int e = 0; e < 16; e += 8) {
              uint4 o;
              o.x = pack_bf16(__uint_as_float(v[e + 0]), __uint_as_float(v[e + 1]));
              o.y = pack_bf16(__uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
              o.z = pack_bf16(__uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
              o.w = pack_bf16(__uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
              *reinterpret_cast<uint4*>(drow + c + e) = o;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(oempty);
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

template <BwdPass PASS, int D1, int D2, int SEL>
cudaError_t launch_t(const BwdSplitParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = SplitLayout<PASS, D1, D2>::alloc;
  auto kern = streamkl_bwd_split_kernel<PASS, D1, D2, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <BwdPass PASS, int SEL>
cudaError_t launch_sel(const BwdSplitParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<PASS, 128, 128, SEL>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<PASS, 128, 64, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<PASS, 64, 128, SEL>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<PASS, 64, 64, SEL>(p, grid, stream);
  return cudaErrorInvalidValue;
}

// The instance is chosen by the outputs this pass writes (the page's gradient
// configurations: one side only, or both).
template <BwdPass PASS>
cudaError_t launch_pass(const BwdSplitParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  const int sel = (p.out1 ? 1 : 0) | (p.out2 ? 2 : 0);
  if (sel == 1) return launch_sel<PASS, 1>(p, d1, d2, grid, stream);
  if (sel == 2) return launch_sel<PASS, 2>(p, d1, d2, grid, stream);
  if (sel == 3) return launch_sel<PASS, 3>(p, d1, d2, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_bwd_split(const BwdSplitParams& p, BwdPass pass, int d1, int d2, int grid,
                             cudaStream_t stream) {
  return pass == BwdPass::kDK ? launch_pass<BwdPass::kDK>(p, d1, d2, grid, stream)
                              : launch_pass<BwdPass::kDQ>(p, d1, d2, grid, stream);
}

}  // namespace skl
