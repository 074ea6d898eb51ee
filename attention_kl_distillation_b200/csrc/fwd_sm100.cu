// fwd_sm100.cu -- fused single-pass attention-KL forward for sm_100a.
//
// StreamKL summary page, "Metodologia" section 1: each query row keeps five
// running scalars (m1, m2, l1, l2, acc) while key tiles stream through on-chip
// memory, and finishes with L = acc/l1 + LSE2 - LSE1, LSE_t = m_t + log l_t.
// Key tiles past the causal frontier are never loaded or multiplied.
//
// B200 mapping (one CTA per SM, persistent):
//   work unit   (bh, 128-row query tile)
//   warp 0      TMA producer: per unit the 128 query rows of Q1/Q2 into a
//               staging buffer, per key tile K1/K2 into a ring of up to six
//               stages (128-byte swizzle, no multicast)
//   warp 1      TMEM owner and UMMA issuer: per key tile S1 = Q1 K1^T and
//               S2 = Q2 K2^T (tcgen05.mma kind::f16, M = 128 rows, N = 128
//               keys, fp32 accumulators).  Q lives in TMEM as the A operand,
//               K in shared memory as B.  At the start of a unit this thread
//               copies the staged Q rows into TMEM (tcgen05.cp) once the last
//               products of the previous unit have read the old ones; the
//               staging buffer is refilled for the next unit meanwhile.  The S
//               products rotate through three TMEM slots: S1 of the next key
//               tile is queued behind S2 of this one while the reduction warps
//               read this one, so the tensor pipe does not drain between key
//               tiles.
//   warps 2..17 four reduction warpgroups, each owning 32 of the 128 keys of
//               every key tile: thread r owns query row r (TMEM lane r).  At
//               each key tile each thread loads its
//               32 + 32 logits with tcgen05.ld, frees the slots and applies the
//               online update in registers (exp2 on the MUFU pipe, the softmax
//               scale folded into the exponent argument, packed f32x2
//               arithmetic elsewhere).  The four key parts of a row keep
//               separate running states and merge at the end of the unit.
//               Four reduction warps per SM sub-partition hide each other's
//               latencies.
// The accumulator acc is one fp32 per row: there is no PV product and no
// output tile.  TMEM: S slots [0,128) [128,256) [256,384); Q1/Q2 as bf16 A
// operands [384, 384 + (d1 + d2)/2).
//
// Units are visited longest first (the last query tiles of a causal problem
// see the most keys) and dealt to CTAs in a snake order, an approximation of
// longest-processing-time scheduling.  When a head has at least one query tile
// per SM, heads run one after another so that concurrent CTAs share its key
// tiles in L2; otherwise the units of one query tile across all heads run
// together.
#include "kernels.h"
#include "sm100.cuh"

#include <cmath>

namespace skl {
namespace {

constexpr int BQ = kFwdBQ;
constexpr int BK = kFwdBK;
constexpr int NH = 4;        // reduction warpgroups, each owning KH keys of every key tile
constexpr int KH = BK / NH;
constexpr int NSLOT = 3;     // TMEM slots the S products rotate through
constexpr int NTHREADS = 64 + NH * 128;
constexpr float kLn2 = 0.6931471805599453f;

template <int D1, int D2>
struct FwdLayout {
  static constexpr int q1_bytes = BQ * D1 * 2;  // staged query rows, TMA -> tcgen05.cp
  static constexpr int q2_bytes = BQ * D2 * 2;
  static constexpr int k1_bytes = BK * D1 * 2;
  static constexpr int k2_bytes = BK * D2 * 2;
  static constexpr int stage_bytes = k1_bytes + k2_bytes;
  static constexpr int handover_bytes = (NH - 1) * 5 * BQ * 4;
  static constexpr int q_off = 0;
  static constexpr int k_off = q_off + q1_bytes + q2_bytes;
  static constexpr int ks_fit = (232448 - 1024 - 512 - handover_bytes - k_off) / stage_bytes;
  static constexpr int KSTAGES = ks_fit > 6 ? 6 : ks_fit;
  static constexpr int bar_off = k_off + KSTAGES * stage_bytes;
  // barriers: qsfull, qsempty, qdone, kfull[KS][2], kempty[KS][2], sfull[NSLOT],
  // sempty[NSLOT], drain
  static constexpr int nbar = 4 + 4 * KSTAGES + 2 * NSLOT;
  static constexpr int misc_off = bar_off + nbar * 8;
  static constexpr int part_off = misc_off + 16;  // key-part states [NH-1][5][BQ] fp32
  static constexpr int total = part_off + handover_bytes;
  static constexpr int alloc = total + 1024;  // slack to align the base to 1024 B
  static_assert(KSTAGES >= 2, "key ring too shallow");
  static_assert(alloc <= 232448, "shared memory budget exceeded");
  static_assert(k1_bytes % 1024 == 0 && k2_bytes % 1024 == 0 && q1_bytes % 1024 == 0 &&
                    q2_bytes % 1024 == 0,
                "tiles must keep 1024-byte alignment for the 128B swizzle atoms");
  // TMEM columns
  __host__ __device__ static constexpr uint32_t s_col(int slot) { return slot * BK; }
  static constexpr uint32_t q_col = NSLOT * BK;  // Q1; Q2 at +D1/2
  static_assert(NSLOT * BK + (D1 + D2) / 2 <= 512, "TMEM budget exceeded");
};

// Rotation of the S products through the TMEM slots.  Counted over the CTA's
// whole run, product k (S1 of a key tile, then its S2) uses slot k mod NSLOT;
// a slot's two barriers complete one phase per use.  The issuer and the
// reduction warps step their own copies through the same sequence.
struct SlotRing {
  int s = 0;
  uint32_t ph = 0;  // bit i: parity of slot i's current use
  __device__ __forceinline__ int slot() const { return s; }
  __device__ __forceinline__ uint32_t parity() const { return (ph >> s) & 1u; }
  __device__ __forceinline__ void advance() {
    ph ^= 1u << s;
    s = (s == NSLOT - 1) ? 0 : s + 1;
  }
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
  int bh, q0;
  int kt_lo;    // first key tile of this unit (split-K chunk start; 0 without split)
  int nkt;      // end of the key tiles the tile processes (<= kt_lo: none)
  int kt_mask;  // key tiles [kt_mask, nkt) need element masks
  int split;    // key split index (0 without split)
};

__device__ __forceinline__ Unit decode_unit(const FwdParams& p, int u) {
  const int nqb = (p.NQ + BQ - 1) / BQ;
  Unit w;
  w.split = 0;
  if (p.nsplit > 1) {
    w.split = u % p.nsplit;
    u /= p.nsplit;
  }
  // Heads in groups of p.head_group: within a group, query tiles longest first
  // and heads innermost.  With one head per group, the CTAs running at one time
  // all stream the same head's key tiles at about the same time, so long
  // problems read K from L2 instead of HBM.  With every head in one group, the
  // longest units of all heads come first, which keeps the last wave short.
  const int G = max(1, min(p.head_group, p.BH));
  const int g = u / (G * nqb);
  const int gsize = min(G, p.BH - g * G);
  const int r = u - g * G * nqb;
  w.bh = g * G + r % gsize;
  w.q0 = (nqb - 1 - r / gsize) * BQ;  // longest (last) query tiles first
  const int nkt_all = (p.NK + BK - 1) / BK;
  const int off = p.NK - p.NQ;
  w.kt_lo = p.nsplit > 1 ? w.split * p.kt_chunk : 0;
  const int kt_hi = p.nsplit > 1 ? min(nkt_all, w.kt_lo + p.kt_chunk) : nkt_all;
  w.nkt = kt_hi;
  w.kt_mask = (p.NK % BK) ? nkt_all - 1 : nkt_all;
  if (p.causal) {
    const int last = min(w.q0 + BQ - 1, p.NQ - 1) + off;  // last key any row of the tile sees
    w.nkt = min(kt_hi, last / BK + 1);
    w.kt_mask = min(w.kt_mask, (w.q0 + off + 1) / BK);  // first tile the first row cannot fully see
  }
  return w;
}

struct RowState {
  float m1, m2, l1, l2, acc;
};

// One key tile (this warpgroup's KH keys of it) of the online update for one
// row.  a/b hold the raw fp32 products <Q1_i, K1_j> and <Q2_i, K2_j>; c1/c2
// fold the softmax scale and log2(e).  With MASK, only the first nv keys are
// visible.
template <bool MASK>
__device__ __forceinline__ void tile_update(const uint32_t (&a)[KH], const uint32_t (&b)[KH],
                                            float c1, float c2, int nv, RowState& st) {
  float mx1[4], mx2[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) mx1[k] = mx2[k] = -INFINITY;
#pragma unroll
  for (int j = 0; j < KH; j += 2) {
    float v1a = __uint_as_float(a[j]), v1b = __uint_as_float(a[j + 1]);
    float v2a = __uint_as_float(b[j]), v2b = __uint_as_float(b[j + 1]);
    if (MASK) {
      if (j >= nv) v1a = v2a = -INFINITY;
      if (j + 1 >= nv) v1b = v2b = -INFINITY;
    }
    const int k = (j >> 1) & 3;
    mx1[k] = max3(mx1[k], v1a, v1b);
    mx2[k] = max3(mx2[k], v2a, v2b);
  }
  const float tmx1 = fmaxf(max3(mx1[0], mx1[1], mx1[2]), mx1[3]);
  const float tmx2 = fmaxf(max3(mx2[0], mx2[1], mx2[2]), mx2[3]);
  const float m1n = fmaxf(st.m1, tmx1 * c1);
  const float m2n = fmaxf(st.m2, tmx2 * c2);
  // A row that has seen no key yet keeps m = -inf; shift by 0 instead so that
  // no inf - inf appears.  (Every valid row sees key 0 in its first tile.)
  const float m1u = (m1n == -INFINITY) ? 0.f : m1n;
  const float m2u = (m2n == -INFINITY) ? 0.f : m2n;
  const float2 C1 = make_float2(c1, c1), C2 = make_float2(c2, c2);
  const float2 M1 = make_float2(-m1u, -m1u), M2 = make_float2(-m2u, -m2u);
  const float2 NEG1 = make_float2(-1.f, -1.f);
  float2 sp1[2], sp2[2], sd[2];
#pragma unroll
  for (int k = 0; k < 2; ++k) sp1[k] = sp2[k] = sd[k] = make_float2(0.f, 0.f);
#pragma unroll
  for (int j = 0; j < KH; j += 2) {
    const float2 v1 = make_float2(__uint_as_float(a[j]), __uint_as_float(a[j + 1]));
    const float2 v2 = make_float2(__uint_as_float(b[j]), __uint_as_float(b[j + 1]));
    float2 t1 = __ffma2_rn(v1, C1, M1);  // log2 of the unnormalised teacher weight
    float2 t2 = __ffma2_rn(v2, C2, M2);
    float2 p1 = make_float2(ex2(t1.x), ex2(t1.y));
    float2 p2 = make_float2(ex2(t2.x), ex2(t2.y));
    if (MASK) {
      if (j >= nv) p1.x = p2.x = t1.x = t2.x = 0.f;
      if (j + 1 >= nv) p1.y = p2.y = t1.y = t2.y = 0.f;
    }
    const int k = (j >> 1) & 1;
    sp1[k] = __fadd2_rn(sp1[k], p1);
    sp2[k] = __fadd2_rn(sp2[k], p2);
    sd[k] = __ffma2_rn(p1, __ffma2_rn(t2, NEG1, t1), sd[k]);  // p1 * (t1 - t2)
  }
  const float s1 = (sp1[0].x + sp1[0].y) + (sp1[1].x + sp1[1].y);
  const float s2 = (sp2[0].x + sp2[0].y) + (sp2[1].x + sp2[1].y);
  const float d = (sd[0].x + sd[0].y) + (sd[1].x + sd[1].y);
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
  constexpr int KS = Lay::KSTAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bar_off);
  uint64_t* qsfull = bars + 0;     // a unit's Q rows have landed in the staging buffer
  uint64_t* qsempty = qsfull + 1;  // they have been copied into TMEM
  uint64_t* qdone = qsempty + 1;   // the UMMAs of the previous unit have read Q in TMEM
  // [KS][2]: the K1 and K2 halves of a stage are filled and freed separately,
  // so K1 of a later key tile is in flight as soon as S1 has read this one
  uint64_t* kfull = qdone + 1;
  uint64_t* kempty = kfull + 2 * KS;
  uint64_t* sfull = kempty + 2 * KS;  // [NSLOT]
  uint64_t* sempty = sfull + NSLOT;   // [NSLOT]
  uint64_t* drain = sempty + NSLOT;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::misc_off);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::misc_off + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  WaitCtl ctl{abort_flag, p.status, p.wait_limit_ns};

  if (threadIdx.x == 0) {
    *abort_flag = 0;
    mbar_init(qsfull, 1);
    mbar_init(qsempty, 1);
    mbar_init(qdone, 1);
    for (int s = 0; s < 2 * KS; ++s) {
      mbar_init(&kfull[s], 1);
      mbar_init(&kempty[s], 1);
    }
    for (int s = 0; s < NSLOT; ++s) {
      mbar_init(&sfull[s], 1);
      mbar_init(&sempty[s], 4 * NH);  // one arrival per reduction warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_desc(&p.tmQ1);
    tma_prefetch_desc(&p.tmQ2);
    tma_prefetch_desc(&p.tmK1);
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

  Sched sched{fwd_units(p.BH, p.NQ, p.nsplit), static_cast<int>(gridDim.x),
              static_cast<int>(blockIdx.x), 0};
  uint8_t* q1_s = smem + Lay::q_off;
  uint8_t* q2_s = q1_s + Lay::q1_bytes;
  auto k1_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes; };
  auto k2_s = [&](int s) { return smem + Lay::k_off + s * Lay::stage_bytes + Lay::k1_bytes; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int ks = 0;
      uint32_t kph = 0, qph = 0;
      uint32_t armed_k[2 * KS] = {};  // last armed phase + 1 (0 = never)
      uint32_t armed_q = 0;
      int u;
      bool ok = true;
      while (ok && sched.next(u)) {
        const Unit w = decode_unit(p, u);
        if (w.nkt <= w.kt_lo) continue;  // split chunk past every row's frontier
        // This unit's query rows (rows past NQ are zero-filled), once the
        // previous unit's rows have been copied out of the staging buffer.
        if (!(ok = mbar_wait(qsempty, qph ^ 1, ctl))) break;
        mbar_arrive_expect_tx(qsfull, Lay::q1_bytes + Lay::q2_bytes);
#pragma unroll
        for (int b = 0; b < D1 / 64; ++b)
          tma_load_3d(q1_s + b * (BQ * 128), &p.tmQ1, qsfull, b * 64, w.q0, w.bh);
#pragma unroll
        for (int b = 0; b < D2 / 64; ++b)
          tma_load_3d(q2_s + b * (BQ * 128), &p.tmQ2, qsfull, b * 64, w.q0, w.bh);
        armed_q = qph + 1;
        qph ^= 1;
        for (int kt = w.kt_lo; kt < (p.withhold_keys ? w.kt_lo : w.nkt); ++kt) {
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
        if (armed_q) mbar_wait(qsfull, armed_q - 1, dctl);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BQ, BK);
      const uint32_t a1 = tmem_base + Lay::q_col, a2 = a1 + D1 / 2;
      const uint64_t q1sd = sdesc_sw128(smem_u32(q1_s), 16, 1024);
      const uint64_t q2sd = sdesc_sw128(smem_u32(q2_s), 16, 1024);
      int ks = 0;
      uint32_t kph = 0, qsph = 0, qdph = 0;
      bool first = true;
      SlotRing ring;
      int u;
      bool ok = true;
      while (ok && sched.next(u)) {
        const Unit w = decode_unit(p, u);
        if (w.nkt <= w.kt_lo) continue;
        if (!first) {
          // The previous unit's products must have read Q out of TMEM before
          // it is overwritten (a copy is not ordered after earlier products).
          umma_commit(qdone);
          if (!(ok = mbar_wait(qdone, qdph, ctl))) break;
          qdph ^= 1;
        }
        first = false;
        if (!(ok = mbar_wait(qsfull, qsph, ctl))) break;  // Q rows of this unit staged
        qsph ^= 1;
        tc_fence_after();
        // Staged rows into TMEM, one 16-feature slice per copy at the columns the
        // products read it from; the products issued below see the copies.
#pragma unroll
        for (int kk = 0; kk < D1 / 16; ++kk)
          tmem_cp_128x256b(a1 + kk * 8, sdesc_advance(q1sd, (kk >> 2) * (BQ * 128) + (kk & 3) * 32));
#pragma unroll
        for (int kk = 0; kk < D2 / 16; ++kk)
          tmem_cp_128x256b(a2 + kk * 8, sdesc_advance(q2sd, (kk >> 2) * (BQ * 128) + (kk & 3) * 32));
        umma_commit(qsempty);  // the staging buffer is free once the copies are done
        for (int kt = w.kt_lo; kt < w.nkt; ++kt) {
          // Descriptors built once per stage; each UMMA below costs an add and the
          // MMA itself, so this thread keeps up although it shares its SM
          // sub-partition with four busy reduction warps.
          const uint64_t b1 = sdesc_sw128(smem_u32(k1_s(ks)), 16, 1024);
          const uint64_t b2 = sdesc_sw128(smem_u32(k2_s(ks)), 16, 1024);
          // S1 into the next slot once K1 has landed and the reduction warps
          // have read the slot out
          if (!(ok = mbar_wait(&kfull[2 * ks], kph, ctl))) break;
          if (!(ok = mbar_wait(&sempty[ring.slot()], ring.parity() ^ 1, ctl))) break;
          tc_fence_after();
          {
            const uint32_t d = tmem_base + Lay::s_col(ring.slot());
#pragma unroll
            for (int kk = 0; kk < D1 / 16; ++kk)
              umma_bf16_ts(d, a1 + kk * 8,
                           sdesc_advance(b1, (kk >> 2) * (BK * 128) + (kk & 3) * 32), idesc, kk > 0);
            umma_commit(&sfull[ring.slot()]);
            umma_commit(&kempty[2 * ks]);
            ring.advance();
          }
          if (!(ok = mbar_wait(&kfull[2 * ks + 1], kph, ctl))) break;
          if (!(ok = mbar_wait(&sempty[ring.slot()], ring.parity() ^ 1, ctl))) break;
          tc_fence_after();
          {
            const uint32_t d = tmem_base + Lay::s_col(ring.slot());
#pragma unroll
            for (int kk = 0; kk < D2 / 16; ++kk)
              umma_bf16_ts(d, a2 + kk * 8,
                           sdesc_advance(b2, (kk >> 2) * (BK * 128) + (kk & 3) * 32), idesc, kk > 0);
            umma_commit(&sfull[ring.slot()]);
            umma_commit(&kempty[2 * ks + 1]);
            ring.advance();
          }
          if (++ks == KS) {
            ks = 0;
            kph ^= 1;
          }
        }
        if (!ok) break;
      }
      // Every UMMA issued by this thread completes before TMEM is released.
      umma_commit(drain);
      volatile int zero = 0;
      WaitCtl dctl{&zero, p.status, p.wait_limit_ns};
      mbar_wait(drain, 0, dctl);
    }
  } else {
    // ------------------------------------------------------------ reduction
    const int hf = (warp - 2) >> 2;  // which KH keys of every key tile this warpgroup owns
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t tlane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    float* part = reinterpret_cast<float*>(smem + Lay::part_off);
    const int off = p.NK - p.NQ;
    SlotRing ring;
    int u;
    bool ok = true;
    while (ok && sched.next(u)) {
      const Unit w = decode_unit(p, u);
      if (w.nkt <= w.kt_lo) continue;
      const int i_abs = w.q0 + row;
      const int lim = p.causal ? min(p.NK, i_abs + off + 1) : p.NK;  // visible keys [0, lim)
      RowState st{-INFINITY, -INFINITY, 0.f, 0.f, 0.f};
      for (int kt = w.kt_lo; kt < w.nkt; ++kt) {
        uint32_t a[KH], b[KH];
        const int sa = ring.slot();
        if (!(ok = mbar_wait(&sfull[sa], ring.parity(), ctl))) break;
        ring.advance();
        tc_fence_after();
        tmem_ld_32x32b<KH>(tlane + Lay::s_col(sa) + hf * KH, a);
        const int sb = ring.slot();
        if (!(ok = mbar_wait(&sfull[sb], ring.parity(), ctl))) break;
        ring.advance();
        tc_fence_after();
        tmem_ld_32x32b<KH>(tlane + Lay::s_col(sb) + hf * KH, b);
        tmem_ld_wait();
        reg_fence(a);
        reg_fence(b);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sempty[sa]);
          mbar_arrive(&sempty[sb]);
        }
        if (kt >= w.kt_mask)
          tile_update<true>(a, b, p.c1, p.c2, lim - kt * BK - hf * KH, st);
        else
          tile_update<false>(a, b, p.c1, p.c2, KH, st);
      }
      if (!ok) break;
      // Merge the key parts of every row (same rescaling as the split-K merge):
      // the other warpgroups hand their states over through shared memory.
      if (hf > 0) {
        float* slot = part + (hf - 1) * 5 * BQ;
        slot[0 * BQ + row] = st.m1;
        slot[1 * BQ + row] = st.m2;
        slot[2 * BQ + row] = st.l1;
        slot[3 * BQ + row] = st.l2;
        slot[4 * BQ + row] = st.acc;
      }
      named_bar_sync(1, NH * 128);
      if (hf == 0) {
#pragma unroll
        for (int o = 0; o < NH - 1; ++o) {
          const float* slot = part + o * 5 * BQ;
          const float om1 = slot[0 * BQ + row], om2 = slot[1 * BQ + row];
          const float m1 = fmaxf(st.m1, om1), m2 = fmaxf(st.m2, om2);
          // a part with no visible key has m = -inf and weight 0; two such
          // parts keep the empty state
          const float fa1 = st.m1 == -INFINITY ? 0.f : ex2(st.m1 - m1);
          const float fb1 = om1 == -INFINITY ? 0.f : ex2(om1 - m1);
          const float fa2 = st.m2 == -INFINITY ? 0.f : ex2(st.m2 - m2);
          const float fb2 = om2 == -INFINITY ? 0.f : ex2(om2 - m2);
          st.l1 = fmaf(st.l1, fa1, slot[2 * BQ + row] * fb1);
          st.l2 = fmaf(st.l2, fa2, slot[3 * BQ + row] * fb2);
          st.acc = fmaf(st.acc, fa1, slot[4 * BQ + row] * fb1);
          st.m1 = m1;
          st.m2 = m2;
        }
      }
      named_bar_sync(1, NH * 128);  // the handover slots may be reused
      if (hf == 0 && i_abs < p.NQ) {
        const size_t o = static_cast<size_t>(w.bh) * p.NQ + i_abs;
        if (p.nsplit > 1) {
          // partial state of this key chunk, merged by streamkl_fwd_merge_kernel
          const size_t rows = static_cast<size_t>(p.BH) * p.NQ;
          float* dst = p.part + static_cast<size_t>(w.split) * 5 * rows + o;
          dst[0 * rows] = st.m1;
          dst[1 * rows] = st.m2;
          dst[2 * rows] = st.l1;
          dst[3 * rows] = st.l2;
          dst[4 * rows] = st.acc;
        } else {
          const float lg1 = lg2(st.l1), lg2v = lg2(st.l2);
          p.LSE1[o] = kLn2 * (st.m1 + lg1);
          p.LSE2[o] = kLn2 * (st.m2 + lg2v);
          p.L[o] = kLn2 * (st.acc / st.l1 + (st.m2 - st.m1) + (lg2v - lg1));
        }
      }
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

// Split-K merge (the page's Split-K variant, section 3): per row, combine the
// partial states of the key chunks that overlap its visible keys,
//   m = max_c m_c,  l = sum_c l_c 2^(m_c - m),  acc = sum_c acc_c 2^(m1_c - m1),
// then finish as the unsplit kernel does.  acc_c holds sum p1 (y1 - y2) with p1
// relative to m1_c, so it rescales with the teacher's factor.
__global__ void streamkl_fwd_merge_kernel(const FwdMergeParams p) {
  const long long rows = static_cast<long long>(p.BH) * p.NQ;
  const int off = p.NK - p.NQ;
  for (long long r = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; r < rows;
       r += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int i = static_cast<int>(r % p.NQ);
    const int lim = p.causal ? min(p.NK, i + off + 1) : p.NK;
    const int nc = min(p.nsplit, (lim + p.kt_chunk * BK - 1) / (p.kt_chunk * BK));
    float m1 = -INFINITY, m2 = -INFINITY;
    for (int c = 0; c < nc; ++c) {
      m1 = fmaxf(m1, p.part[(static_cast<size_t>(c) * 5 + 0) * rows + r]);
      m2 = fmaxf(m2, p.part[(static_cast<size_t>(c) * 5 + 1) * rows + r]);
    }
    float l1 = 0.f, l2 = 0.f, acc = 0.f;
    for (int c = 0; c < nc; ++c) {
      const float* q = p.part + static_cast<size_t>(c) * 5 * rows + r;
      const float f1 = ex2(q[0] - m1), f2 = ex2(q[1 * rows] - m2);  // 0 for an empty chunk
      l1 = fmaf(q[2 * rows], f1, l1);
      l2 = fmaf(q[3 * rows], f2, l2);
      acc = fmaf(q[4 * rows], f1, acc);
    }
    const float lg1 = lg2(l1), lg2v = lg2(l2);
    p.LSE1[r] = kLn2 * (m1 + lg1);
    p.LSE2[r] = kLn2 * (m2 + lg2v);
    p.L[r] = kLn2 * (acc / l1 + (m2 - m1) + (lg2v - lg1));
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

cudaError_t launch_fwd_merge(const FwdMergeParams& p, int num_sms, cudaStream_t stream) {
  streamkl_fwd_merge_kernel<<<num_sms * 4, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdParams& p, int d1, int d2, int grid, cudaStream_t stream) {
  if (d1 == 128 && d2 == 128) return launch_t<128, 128>(p, grid, stream);
  if (d1 == 128 && d2 == 64) return launch_t<128, 64>(p, grid, stream);
  if (d1 == 64 && d2 == 128) return launch_t<64, 128>(p, grid, stream);
  if (d1 == 64 && d2 == 64) return launch_t<64, 64>(p, grid, stream);
  return cudaErrorInvalidValue;
}

}  // namespace skl
