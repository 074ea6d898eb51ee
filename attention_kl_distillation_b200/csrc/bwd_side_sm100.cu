// bwd_side_sm100.cu -- recompute backward of the fused attention-KL for sm_100a,
// one gradient side per launch with 128-key steps.
//
// Same arithmetic as bwd_qt_sm100.cu (StreamKL summary page, "Metodologia"
// section 2; the page's two gradient configurations, "Calcolo del Gradiente"):
// a work unit is one 128-query tile, dQ_t stays in TMEM over the unit's key
// steps and dK_t goes through fp32 reductions into the workspace.  This kernel
// forms and contracts one side t only (the teacher's dS1 or the student's
// dS2); both sides are two launches.
//
// Why: a single issuing thread needs about as long for an M128 N64 UMMA as for
// an N128 one, so the products of 64-key steps run at half the tensor rate.
// With one side per CTA, TMEM holds S1 and S2 of a 128-key step (256 columns),
// dQ_t (d_t) and dK_t^T (128), and every product is N = 128: per 64 keys of
// one side, 8 S products, 4 dQ_t and 4 dK_t^T instead of 16, 4 and 8.
//
// B200 mapping (one CTA per SM, persistent, units handed out dynamically):
//   work unit   (bh, 128-query tile); inner loop over the 128-key steps it sees
//   warp 0      TMA producer: Q1/Q2 tile per unit, per step the keys of this
//               side (K_t, read by S and dQ_t, free once the step is done) into
//               a ring of up to four stages and the other side's keys (read by
//               S only, free once S is done) into a shorter ring
//   warp 1      TMEM owner and UMMA issuer, per step:
//                 S1 = Q1 K1^T, S2 = Q2 K2^T                (M=128, N=128 keys)
//                 dQ_t += dS_t K_t                          (M=128, N=d_t)
//                 dK_t^T = Q_t^T dS_t                       (M=d_t, N=128 keys)
//   warps 2..9  two dS warpgroups, each for 64 of the 128 keys of a step, read
//               from TMEM in two chunks of 32; thread r owns query row r
//   warps 10..13 dK warpgroup: dK_t^T (thread = feature) reduced into the fp32
//               workspace; at the end of a unit dQ_t to bf16.
// TMEM (512 columns): S1 [0,128) S2 [128,256) dQ_t [256,256+d_t) dK_t^T [384,512).
// One commit per step, on this side's key-stage barrier, tells the producer,
// the dS warps (the dS tile is free) and the dK warps (dK_t^T is ready).
#include "kernels.h"
#include "sm100.cuh"

#include <cuda_bf16.h>

#include <cmath>

namespace skl {
namespace {

constexpr int RQ = kBwdQtRows;  // queries per unit
constexpr int CK = 128;         // keys per step
constexpr int NDS = 2;          // dS warpgroups
constexpr int KPW = CK / NDS;   // keys of a step per dS warpgroup
constexpr int KCH = 32;         // keys per TMEM chunk a dS thread holds at once
constexpr int DK_WARP0 = 2 + 4 * NDS;
constexpr int NTHREADS = (DK_WARP0 + 4) * 32;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kColS1 = 0, kColS2 = 128, kColDQ = 256, kColDK = 384;

template <int D1, int D2, int SIDE>
struct SideLayout {
  static constexpr int DT = SIDE == 1 ? D1 : D2;  // this side's head dimension
  static constexpr int DO = SIDE == 1 ? D2 : D1;  // the other side's
  static constexpr int q1_bytes = RQ * D1 * 2;
  static constexpr int q2_bytes = RQ * D2 * 2;
  static constexpr int kt_bytes = CK * DT * 2;    // one stage of this side's keys
  static constexpr int ko_bytes = CK * DO * 2;    // one stage of the other side's keys
  static constexpr int ds_bytes = RQ * CK * 2;  // dS_t, bf16 [128 queries][128 keys], two 64-key chunks
  static constexpr int fixed_bytes = q1_bytes + q2_bytes + ds_bytes + 1024 + 512;
  static constexpr bool fits(int nt, int no) {
    return fixed_bytes + nt * kt_bytes + no * ko_bytes <= 232448;
  }
  // This side's keys stay from S of a step to its contractions, so their ring
  // is the deeper one: the stage for step t+1 was freed by step t-2.  The other
  // side's keys are free once S is done.
  static constexpr int NO = fits(3, 2) ? 2 : 1;
  static constexpr int NT = fits(4, NO) ? 4 : 3;
  static constexpr int q1_off = 0;
  static constexpr int q2_off = q1_off + q1_bytes;
  static constexpr int ds_off = q2_off + q2_bytes;
  static constexpr int kt_off = ds_off + ds_bytes;
  static constexpr int ko_off = kt_off + NT * kt_bytes;
  static constexpr int bar_off = ko_off + NO * ko_bytes;
  // qfull qempty kfullT[NT] kemptyT[NT] kfullO[NO] kemptyO[NO] sfull sempty dsfull
  // dkempty dqfull dqempty ufull[2] uempty[2] drain
  static constexpr int nbar = 2 + 2 * NT + 2 * NO + 4 + 2 + 4 + 1;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int total = misc_off + 32;
  static constexpr int alloc = total + 1024;
  static_assert(fits(NT, NO), "key rings too deep");
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(q1_bytes % 1024 == 0 && q2_bytes % 1024 == 0 && kt_bytes % 1024 == 0 &&
                    ko_bytes % 1024 == 0,
                "operand tiles must stay 1024-byte aligned");
};

struct UnitS {
  int bh, q0, nsteps;
  int kmask;  // key steps from kmask on need element masks
  int rot;    // iteration t visits key step (t + rot) mod nsteps
  __device__ __forceinline__ int step(int t) const {
    int r = t + rot;
    if (r >= nsteps) r -= nsteps;
    return r;
  }
};

__device__ __forceinline__ UnitS decode_unit(const BwdSideParams& p, int u) {
  const int nqt = (p.NQ + RQ - 1) / RQ;
  UnitS w;
  w.bh = u / nqt;
  w.q0 = (nqt - 1 - u % nqt) * RQ;  // within a head, the query tiles that see most keys first
  const int off = p.NK - p.NQ;
  int nk = p.NK, full = p.NK;
  if (p.causal) {
    nk = min(p.NK, min(w.q0 + RQ - 1, p.NQ - 1) + off + 1);
    full = min(full, w.q0 + off + 1);
  }
  w.nsteps = (nk + CK - 1) / CK;
  w.kmask = full / CK;
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

// This thread's query row (see bwd_qt_sm100.cu): u_t = c_t S_t + b_t = log2 P_t,
// s1 dS1 = P1 (gl (u1 - u2) + gn), s2 dS2 = g2 (P2 - P1).
struct RowRec {
  float b1, b2, gl, gn, g2;
};

// s_t dS_t for one query row and KCH keys into bf16 pairs.  SIDE 1 needs the
// student only through u2 (no P2 exponential).  MASK: column c visible iff c <= last.
template <int SIDE, bool MASK>
__device__ __forceinline__ void form_chunk(const uint32_t (&s1)[KCH], const uint32_t (&s2)[KCH],
                                           const RowRec& rr, float c1, float c2, int last,
                                           uint32_t* w) {
  const float2 C1 = make_float2(c1, c1), C2 = make_float2(c2, c2);
  const float2 B1 = make_float2(rr.b1, rr.b1), B2 = make_float2(rr.b2, rr.b2);
  const float2 GL = make_float2(rr.gl, rr.gl), GN = make_float2(rr.gn, rr.gn);
  const float2 G2v = make_float2(rr.g2, rr.g2);
  const float2 NEG1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int i = 0; i < KCH; i += 2) {
    const float2 S1 = make_float2(__uint_as_float(s1[i]), __uint_as_float(s1[i + 1]));
    const float2 S2 = make_float2(__uint_as_float(s2[i]), __uint_as_float(s2[i + 1]));
    const float2 u1 = __ffma2_rn(S1, C1, B1);
    const float2 u2 = __ffma2_rn(S2, C2, B2);
    const float2 P1 = make_float2(ex2(u1.x), ex2(u1.y));
    float2 d;
    if (SIDE == 1) {
      d = __fmul2_rn(P1, __ffma2_rn(__ffma2_rn(u2, NEG1, u1), GL, GN));
    } else {
      const float2 P2 = make_float2(ex2(u2.x), ex2(u2.y));
      d = __fmul2_rn(__ffma2_rn(P1, NEG1, P2), G2v);
    }
    if (MASK) {
      d.x = i <= last ? d.x : 0.f;
      d.y = i + 1 <= last ? d.y : 0.f;
    }
    w[i / 2] = pack_bf16(d.x, d.y);
  }
}

template <bool FULL>
__device__ __forceinline__ void red_dk(float* base, int ldk, const uint32_t (&v)[32], int nvalid) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if (FULL || i < nvalid) atomicAdd(base + i * ldk, __uint_as_float(v[i]));
}

template <int D1, int D2, int SIDE>
__global__ void __launch_bounds__(NTHREADS, 1)
    streamkl_bwd_side_kernel(const __grid_constant__ BwdSideParams p) {
  constexpr int DT = SIDE == 1 ? D1 : D2;
  constexpr int DO = SIDE == 1 ? D2 : D1;
  using Lay = SideLayout<D1, D2, SIDE>;
  constexpr int NT = Lay::NT, NO = Lay::NO;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* qfull = bars + 0;
  uint64_t* qempty = bars + 1;
  uint64_t* kfullT = bars + 2;        // [NT] this side's keys
  uint64_t* kemptyT = kfullT + NT;    // [NT] completes when the step's products are done
  uint64_t* kfullO = kemptyT + NT;    // [NO] the other side's keys
  uint64_t* kemptyO = kfullO + NO;    // [NO] completes when S is done
  uint64_t* sfull = kemptyO + NO;
  uint64_t* sempty = sfull + 1;
  uint64_t* dsfull = sempty + 1;
  uint64_t* dkempty = dsfull + 1;
  uint64_t* dqfull = dkempty + 1;
  uint64_t* dqempty = dqfull + 1;
  uint64_t* ufull = dqempty + 1;   // [2]
  uint64_t* uempty = ufull + 2;    // [2]
  uint64_t* drain = uempty + 2;
  const CUtensorMap* tmKT = SIDE == 1 ? &p.tmK1 : &p.tmK2;
  const CUtensorMap* tmKO = SIDE == 1 ? &p.tmK2 : &p.tmK1;
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
    for (int s = 0; s < NT; ++s) {
      mbar_init(&kfullT[s], 1);
      mbar_init(&kemptyT[s], 1);
    }
    for (int s = 0; s < NO; ++s) {
      mbar_init(&kfullO[s], 1);
      mbar_init(&kemptyO[s], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(sempty, 4 * NDS);
    mbar_init(dsfull, 4 * NDS);
    mbar_init(dkempty, 4);
    mbar_init(dqfull, 1);
    mbar_init(dqempty, 4);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ufull[s], 1);
      mbar_init(&uempty[s], 1 + 4 * NDS + 4);
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

  const int total = bwd_qt_units(p.BH, p.NQ);
  uint8_t* q1_s = smem + Lay::q1_off;
  uint8_t* q2_s = smem + Lay::q2_off;
  uint8_t* ds_s = smem + Lay::ds_off;
  auto kt_s = [&](int s) { return smem + Lay::kt_off + s * Lay::kt_bytes; };
  auto ko_s = [&](int s) { return smem + Lay::ko_off + s * Lay::ko_bytes; };
  const int off = p.NK - p.NQ;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int us = 0, kst = 0, kso = 0;
      uint32_t uph = 0, qph = 0, kpht = 0, kpho = 0;
      uint32_t armed_q = 0, armedT[NT] = {}, armedO[NO] = {};
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
        const UnitS w = decode_unit(p, u);
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
          // This side's keys first: their deeper ring was freed steps ago, so the
          // load is issued before the producer blocks on the other side's
          // single-stage ring, which S of the previous step frees.
          if (!(ok = mbar_wait(&kemptyT[kst], kpht ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfullT[kst], Lay::kt_bytes);
#pragma unroll
          for (int b = 0; b < DT / 64; ++b)
            tma_load_3d(kt_s(kst) + b * (CK * 128), tmKT, &kfullT[kst], b * 64, k0, w.bh);
          armedT[kst] = kpht + 1;
          if (++kst == NT) {
            kst = 0;
            kpht ^= 1;
          }
          if (!(ok = mbar_wait(&kemptyO[kso], kpho ^ 1, ctl))) break;
          mbar_arrive_expect_tx(&kfullO[kso], Lay::ko_bytes);
#pragma unroll
          for (int b = 0; b < DO / 64; ++b)
            tma_load_3d(ko_s(kso) + b * (CK * 128), tmKO, &kfullO[kso], b * 64, k0, w.bh);
          armedO[kso] = kpho + 1;
          if (++kso == NO) {
            kso = 0;
            kpho ^= 1;
          }
        }
        if (!ok) break;
        next = static_cast<int>(gridDim.x) + atomicAdd(p.counter, 1);
      }
      if (!ok) {
        volatile int zero = 0;
        WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
        if (armed_q) mbar_wait(qfull, armed_q - 1, dctl);
        for (int s = 0; s < NT; ++s)
          if (armedT[s]) mbar_wait(&kfullT[s], armedT[s] - 1, dctl);
        for (int s = 0; s < NO; ++s)
          if (armedO[s]) mbar_wait(&kfullO[s], armedO[s] - 1, dctl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(RQ, CK);          // S: M=128 queries, N=128 keys
      constexpr uint32_t idQ = idesc_bf16(RQ, DT, 0, 1);    // dQ_t: B = K_t MN-major
      constexpr uint32_t idK = idesc_bf16(DT, CK, 1, 1);    // dK_t^T: A = Q_t MN-major, B = dS MN-major
      const uint32_t q1a = smem_u32(q1_s), q2a = smem_u32(q2_s), dsa = smem_u32(ds_s);
      const uint64_t q1d = sdesc_sw128(q1a, 16, 1024), q2d = sdesc_sw128(q2a, 16, 1024);
      // Q_t read MN-major and dS read both ways: 64-element chunks 16 KB apart
      const uint64_t qtm = sdesc_sw128(SIDE == 1 ? q1a : q2a, RQ * 128, 1024);
      const uint64_t dsk = sdesc_sw128(dsa, 16, 1024);
      const uint64_t dsm = sdesc_sw128(dsa, RQ * 128, 1024);
      int us = 0, kst_s = 0, kso_s = 0, kst_r = 0;
      uint32_t uph = 0, qph = 0, kpht_s = 0, kpho_s = 0, sph = 0, dsph = 0, dkph = 0, dqph = 0;
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
        const UnitS w = decode_unit(p, u);
        if (!(ok = mbar_wait(qfull, qph, ctl))) break;
        qph ^= 1;
        auto issue_s = [&]() -> bool {
          if (!mbar_wait(&kfullO[kso_s], kpho_s, ctl)) return false;
          if (!mbar_wait(&kfullT[kst_s], kpht_s, ctl)) return false;
          if (!mbar_wait(sempty, sph ^ 1, ctl)) return false;
          tc_fence_after();
          const uint64_t ktd = sdesc_sw128(smem_u32(kt_s(kst_s)), 16, 1024);
          const uint64_t kod = sdesc_sw128(smem_u32(ko_s(kso_s)), 16, 1024);
          const uint64_t k1d = SIDE == 1 ? ktd : kod;
          const uint64_t k2d = SIDE == 1 ? kod : ktd;
#pragma unroll
          for (int kk = 0; kk < D1 / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (RQ * 128) + (kk & 3) * 32;
            umma_bf16_ss(tmem_base + kColS1, sdesc_advance(q1d, o), sdesc_advance(k1d, o), idS,
                         kk > 0);
          }
#pragma unroll
          for (int kk = 0; kk < D2 / 16; ++kk) {
            const uint32_t o = (kk >> 2) * (RQ * 128) + (kk & 3) * 32;
            umma_bf16_ss(tmem_base + kColS2, sdesc_advance(q2d, o), sdesc_advance(k2d, o), idS,
                         kk > 0);
          }
          umma_commit(sfull);
          umma_commit(&kemptyO[kso_s]);  // the other side's keys are not needed after S
          sph ^= 1;
          if (++kso_s == NO) {
            kso_s = 0;
            kpho_s ^= 1;
          }
          if (++kst_s == NT) {
            kst_s = 0;
            kpht_s ^= 1;
          }
          return true;
        };
        if (!(ok = issue_s())) break;
        for (int t = 0; t < w.nsteps && ok; ++t) {
          if (t + 1 < w.nsteps && !(ok = issue_s())) break;
          if (!(ok = mbar_wait(dsfull, dsph, ctl))) break;
          dsph ^= 1;
          if (t == 0) {  // the previous unit's dQ has been read out of TMEM
            if (!(ok = mbar_wait(dqempty, dqph ^ 1, ctl))) break;
            dqph ^= 1;
          }
          tc_fence_after();
          // dQ_t += (s_t dS_t) K_t: A = dS K-major (two 64-key chunks 16 KB apart),
          // B = K_t read MN-major (64-feature chunks 16 KB apart), 8 K16 steps.
          const uint64_t ktm = sdesc_sw128(smem_u32(kt_s(kst_r)), CK * 128, 1024);
          const uint32_t acc0 = t > 0;
          if (p.want_dq) {
#pragma unroll
            for (int kk = 0; kk < CK / 16; ++kk)
              umma_bf16_ss(tmem_base + kColDQ, sdesc_advance(dsk, (kk >> 2) * (RQ * 128) + (kk & 3) * 32),
                           sdesc_advance(ktm, kk * 2048), idQ, kk > 0 ? 1u : acc0);
          }
          // dK_t^T = Q_t^T (s_t dS_t): A = Q_t MN-major, B = dS MN-major, 8 K16 steps
          // over the 128 queries.
          if (!(ok = mbar_wait(dkempty, dkph ^ 1, ctl))) break;
          dkph ^= 1;
          tc_fence_after();
          if (p.want_dk) {
#pragma unroll
            for (int kk = 0; kk < RQ / 16; ++kk)
              umma_bf16_ss(tmem_base + kColDK, sdesc_advance(qtm, kk * 2048),
                           sdesc_advance(dsm, kk * 2048), idK, kk > 0);
          }
          umma_commit(&kemptyT[kst_r]);  // step done: keys, dS tile, dK_t^T
          if (++kst_r == NT) kst_r = 0;
        }
        if (!ok) break;
        umma_commit(dqfull);
        umma_commit(qempty);
      }
      umma_commit(drain);
      volatile int zero = 0;
      WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
      mbar_wait(drain, 0, dctl);
    }
  } else if (warp < DK_WARP0) {
    // ------------------------------------------------------------ dS warpgroups
    const int part = (warp - 2) >> 2;  // keys [part*KPW, part*KPW + KPW) of each step
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t dsrow = smem_u32(ds_s) + part * (RQ * 128) + static_cast<uint32_t>(r) * 128;
    int us = 0;
    uint32_t uph = 0, sph = 0;
    int pks = -1;
    uint32_t pkph = 0;
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
      const UnitS w = decode_unit(p, u);
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
      const int lim = (p.causal ? min(p.NK - 1, i + off) : p.NK - 1) - part * KPW;
      for (int t = 0; t < w.nsteps; ++t) {
        const int ks = w.step(t);
        const int k0 = ks * CK;
        const bool masked = ks >= w.kmask;
        if (!(ok = mbar_wait(sfull, sph, ctl))) break;
        sph ^= 1;
        tc_fence_after();
        uint32_t wv[KPW / 2];
#pragma unroll
        for (int c = 0; c < KPW / KCH; ++c) {
          uint32_t a[KCH], b[KCH];
          tmem_ld_32x32b<KCH>(tl + kColS1 + part * KPW + c * KCH, a);
          tmem_ld_32x32b<KCH>(tl + kColS2 + part * KPW + c * KCH, b);
          tmem_ld_wait();
          reg_fence(a);
          reg_fence(b);
          if (c == KPW / KCH - 1) {  // the whole S tile of this step is in registers or formed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sempty);
          }
          if (masked)
            form_chunk<SIDE, true>(a, b, rr, p.c1, p.c2, lim - k0 - c * KCH, wv + c * (KCH / 2));
          else
            form_chunk<SIDE, false>(a, b, rr, p.c1, p.c2, 0, wv + c * (KCH / 2));
        }
        // the dS tile is free once the previous step's products are done
        if (pks >= 0 && !(ok = mbar_wait(&kemptyT[pks], pkph, ctl))) break;
#pragma unroll
        for (int c = 0; c < KPW / 8; ++c) {
          const uint32_t sw = static_cast<uint32_t>((c ^ (r & 7)) << 4);
          st_shared_v4(dsrow + sw, wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
        }
        pks = cks;
        pkph = ckph;
        if (++cks == NT) {
          cks = 0;
          ckph ^= 1;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(dsfull);
      }
      if (!ok) break;
    }
  } else {
    // ------------------------------------------------------------ dK / dQ warpgroup
    const int quarter = warp & 3;
    const uint32_t tl = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    // dK_t^T rows are features: M = 128 puts feature f in lane f; M = 64 puts
    // features 16q..16q+15 in lanes 32q..32q+15.
    const int f = (DT == 128) ? quarter * 32 + lane : (lane < 16 ? quarter * 16 + lane : -1);
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
      const UnitS w = decode_unit(p, u);
      for (int t = 0; t < w.nsteps; ++t) {
        const int k0 = w.step(t) * CK;
        if (!(ok = mbar_wait(&kemptyT[cks], ckph, ctl))) break;
        if (++cks == NT) {
          cks = 0;
          ckph ^= 1;
        }
        tc_fence_after();
        const int nvalid = min(CK, p.NK - k0);
        float* base = p.dKacc + (static_cast<size_t>(w.bh) * p.NK + k0) * p.ldk + p.dk_col + f;
        const bool red = p.want_dk && f >= 0;
        // 128 keys in four chunks of 32: two into registers and reduced, then the
        // last two, the slot released once all four are read
        uint32_t v0[32], v1[32];
        if (p.want_dk) {
          tmem_ld_32x32b_x32(tl + kColDK, v0);
          tmem_ld_32x32b_x32(tl + kColDK + 32, v1);
          tmem_ld_wait();
          reg_fence(v0);
          reg_fence(v1);
        }
        if (red) {
          if (nvalid == CK) {
            red_dk<true>(base, p.ldk, v0, 32);
            red_dk<true>(base + 32 * p.ldk, p.ldk, v1, 32);
          } else {
            red_dk<false>(base, p.ldk, v0, nvalid);
            red_dk<false>(base + 32 * p.ldk, p.ldk, v1, nvalid - 32);
          }
        }
        if (p.want_dk) {
          tmem_ld_32x32b_x32(tl + kColDK + 64, v0);
          tmem_ld_32x32b_x32(tl + kColDK + 96, v1);
          tmem_ld_wait();
          reg_fence(v0);
          reg_fence(v1);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dkempty);
        if (red) {
          if (nvalid == CK) {
            red_dk<true>(base + 64 * p.ldk, p.ldk, v0, 32);
            red_dk<true>(base + 96 * p.ldk, p.ldk, v1, 32);
          } else {
            red_dk<false>(base + 64 * p.ldk, p.ldk, v0, nvalid - 64);
            red_dk<false>(base + 96 * p.ldk, p.ldk, v1, nvalid - 96);
          }
        }
      }
      if (!ok) break;
      // Unit epilogue: dQ_t (thread = query row) to bf16.
      if (!(ok = mbar_wait(dqfull, dqph, ctl))) break;
      dqph ^= 1;
      tc_fence_after();
      const int i = w.q0 + quarter * 32 + lane;
      if (p.want_dq) {
        __nv_bfloat16* dst = p.dQ + (static_cast<size_t>(w.bh) * p.NQ + i) * DT;
#pragma unroll
        for (int c = 0; c < DT; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tl + kColDQ + c, v);
          tmem_ld_wait();
          reg_fence(v);
          if (i < p.NQ) {
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

template <int D1, int D2, int SIDE>
cudaError_t launch_t(const BwdSideParams& p, int grid, cudaStream_t stream) {
  constexpr int smem = SideLayout<D1, D2, SIDE>::alloc;
  auto kern = streamkl_bwd_side_kernel<D1, D2, SIDE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NTHREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int SIDE>
cudaError_t launch_side_t(const BwdSideParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128, SIDE>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64, SIDE>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128, SIDE>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64, SIDE>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_bwd_side(const BwdSideParams& p, int d1, int d2, int side, int grid,
                            cudaStream_t stream) {
  if (side == 1) return launch_side_t<1>(p, d1, d2, grid, stream);
  if (side == 2) return launch_side_t<2>(p, d1, d2, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace skl
