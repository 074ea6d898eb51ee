// kernels.h -- parameter blocks and launchers shared between the C-ABI layer
// (streamkl_api.cu) and the sm_100a kernels.  Internal to libstreamkl.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

namespace skl {

// Rows of Q in one forward tile and work unit (the UMMA M dimension and the
// TMEM lanes).
constexpr int kFwdBQ = 128;
// Keys per forward tile (UMMA N).
constexpr int kFwdBK = 128;

struct FwdParams {
  CUtensorMap tmK1, tmK2;  // 3-D maps over [BH][NK][d], 128-row boxes, 128B swizzle
  CUtensorMap tmQ1, tmQ2;  // [BH][NQ][d], boxes of one query group (transposed kernel)
                           // or of 128 rows (row-tile kernel)
  const __nv_bfloat16* Q1;  // [BH][NQ][d1]
  const __nv_bfloat16* Q2;  // [BH][NQ][d2]
  float* L;
  float* LSE1;
  float* LSE2;
  int BH, NQ, NK, causal;
  float c1, c2;  // s_t * log2(e): logits in the base-2 domain
  int* status;   // device status word
  unsigned long long wait_limit_ns;
  int withhold_keys;  // test hook: the producer issues no key tiles (waits then time out)
  // Split-K: 0 = off.  Otherwise every unit covers key tiles [c*kt_chunk, (c+1)*kt_chunk)
  // of split c < nsplit and writes its rows' partial states to `part`
  // ([nsplit][5][BH*NQ]: m1, m2, l1, l2, acc in the base-2 domain) instead of L/LSE.
  int kt_chunk, nsplit;
  float* part;
  // Row-tile kernel: heads per group of the unit order (1 = heads one after
  // another, BH = all heads interleaved per query tile).
  int head_group;
};

struct FwdMergeParams {
  const float* part;
  float* L;
  float* LSE1;
  float* LSE2;
  int BH, NQ, NK, causal, nsplit, kt_chunk;
};

cudaError_t launch_fwd_merge(const FwdMergeParams& p, int num_sms, cudaStream_t stream);

// Dynamic shared memory the forward kernel needs for head dims (d1, d2).
size_t fwd_smem_bytes(int d1, int d2);

// Launch the forward kernel; returns the launch error.
cudaError_t launch_fwd(const FwdParams& p, int d1, int d2, int grid, cudaStream_t stream);

// Transposed forward for few query rows (keys on the UMMA M axis): problems
// with NQ <= kFwdTMaxNQ use it; the rows form query groups of fwd_t_rows(NQ)
// (the UMMA N), and a work unit is (bh, group, key split).
constexpr int kFwdTMaxNQ = 32;
__host__ __device__ inline int fwd_t_rows(int NQ) { return NQ <= 16 ? 16 : 32; }
__host__ __device__ inline int fwd_t_units(int BH, int NQ, int nsplit = 1) {
  const int nqt = fwd_t_rows(NQ);
  return BH * ((NQ + nqt - 1) / nqt) * (nsplit > 1 ? nsplit : 1);
}
cudaError_t launch_fwd_t(const FwdParams& p, int d1, int d2, int nqt, int grid, cudaStream_t stream);

// Keys per backward work unit (UMMA M of S^T and dK) and queries per step.
constexpr int kBwdBK = 128;
constexpr int kBwdBQ = 64;
// Per-query-row record the backward reads, stored field-major per 64-row step
// ([step][field][64]): -LSE1*log2e, -LSE2*log2e, -L, s1*dL, s2*dL, 3 x pad.
constexpr int kRowRec = 8;

struct BwdParams {
  CUtensorMap tmQ1, tmK1, tmQ2, tmK2;  // Q maps: 64-row boxes; K maps: 128-row boxes
  const float* rowrec;  // [BH][NQpad/64][kRowRec][64], NQpad = NQ rounded up to kBwdBQ
  float* dQacc;         // [BH][NQ][ld] fp32, ld = widths of the selected sides, zeroed first
  __nv_bfloat16* dK1;   // [BH][NK][d1] or null
  __nv_bfloat16* dK2;   // [BH][NK][d2] or null
  int BH, NQ, NK, NQpad, causal;
  int want_dq1, want_dk1, want_dq2, want_dk2;
  float c1, c2;  // s_t * log2(e)
  int* status;
  unsigned long long wait_limit_ns;
};

struct BwdPrepParams {
  const float* L;
  const float* LSE1;
  const float* LSE2;
  const float* dL;
  float* rowrec;        // null: no per-query records (the query-tile kernel reads L/LSE itself)
  float* dQacc;         // the fp32 accumulator to zero (dQ or dK, whichever the kernel reduces)
  long long dqacc_elems;
  int* counters;        // two work-unit counters, zeroed
  int BH, NQ, NQpad;
  float s1, s2;
};

struct BwdConvertParams {
  const float* dQacc;  // fp32 [rows][d1 + d2]
  __nv_bfloat16* dQ1;  // [rows][d1], may be null
  __nv_bfloat16* dQ2;  // [rows][d2], may be null
  long long rows;      // BH * NQ (dQ) or BH * NK (dK)
  int d1, d2;
};

// Query-tile variant of the fused backward: a work unit is one 128-query tile
// (the UMMA M of S and dQ), which visits its visible keys in 64-key steps; dQ
// stays in TMEM for the unit, dK goes through fp32 reductions into dKacc.
constexpr int kBwdQtRows = 128;
constexpr int kBwdQtKeys = 64;

struct BwdQtParams {
  CUtensorMap tmQ1, tmK1, tmQ2, tmK2;  // Q maps: 128-row boxes; K maps: 64-row boxes
  const float* L;       // saved state and upstream gradient, fp32 [BH][NQ]
  const float* LSE1;
  const float* LSE2;
  const float* dL;
  float* dKacc;         // [BH][NK][ld] fp32, ld = widths of the selected sides, zeroed first
  int* counter;         // work-unit counter, zeroed first
  __nv_bfloat16* dQ1;   // [BH][NQ][d1] or null
  __nv_bfloat16* dQ2;   // [BH][NQ][d2] or null
  int BH, NQ, NK, causal;
  int want_dq1, want_dk1, want_dq2, want_dk2;
  float c1, c2;  // s_t * log2(e)
  float s1, s2;
  int* status;
  unsigned long long wait_limit_ns;
};

// sel as for launch_bwd.
cudaError_t launch_bwd_qt(const BwdQtParams& p, int d1, int d2, int sel, int grid,
                          cudaStream_t stream);

// One gradient side per launch, 128-query units and 128-key steps (every
// product N = 128): side 1 forms dS1 and writes dQ1 / reduces dK1, side 2 the
// same for the student.  Both sides are two launches sharing the accumulator.
struct BwdSideParams {
  CUtensorMap tmQ1, tmK1, tmQ2, tmK2;  // 128-row boxes
  const float* L;
  const float* LSE1;
  const float* LSE2;
  const float* dL;
  float* dKacc;         // [BH][NK][ldk] fp32, this side's columns from dk_col, zeroed first
  int ldk, dk_col;
  int* counter;         // work-unit counter of this launch, zeroed first
  __nv_bfloat16* dQ;    // [BH][NQ][d_t] of this side, or null
  int BH, NQ, NK, causal;
  int want_dq, want_dk;
  float c1, c2;  // s_t * log2(e)
  float s1, s2;
  int* status;
  unsigned long long wait_limit_ns;
};

cudaError_t launch_bwd_side(const BwdSideParams& p, int d1, int d2, int side, int grid,
                            cudaStream_t stream);
__host__ __device__ inline int bwd_qt_units(int BH, int NQ) {
  return BH * ((NQ + kBwdQtRows - 1) / kBwdQtRows);
}

// Split backward (two passes of one kernel template): the dK pass streams
// query tiles past resident 128-key tiles, the dQ pass streams key tiles past
// resident 128-query tiles; each accumulates its gradient in TMEM and writes
// it once, with no atomics and no dQ accumulator.
enum class BwdPass : int { kDK = 0, kDQ = 1 };

struct BwdSplitParams {
  CUtensorMap tmR1, tmR2;  // resident operand maps (128-row boxes): K for dK, Q for dQ
  CUtensorMap tmC1, tmC2;  // streamed operand maps (64-row boxes): Q for dK, K for dQ
  const float* rowrec;     // [BH][NQpad/64][kRowRec][64]
  int* counter;            // work-unit counter of this pass (zeroed by the prep kernel)
  __nv_bfloat16* out1;     // dK1 or dQ1 (may be null)
  __nv_bfloat16* out2;     // dK2 or dQ2 (may be null)
  int BH, NQ, NK, NQpad, causal;
  float c1, c2;
  int* status;
  unsigned long long wait_limit_ns;
};

cudaError_t launch_bwd_split(const BwdSplitParams& p, BwdPass pass, int d1, int d2, int grid,
                             cudaStream_t stream);

size_t bwd_smem_bytes(int d1, int d2);
// sel: gradient sides the fused kernel forms -- 1 teacher (dQ1/dK1), 2 student
// (dQ2/dK2), 3 both; the dQ accumulator rows hold the selected sides only.
cudaError_t launch_bwd(const BwdParams& p, int d1, int d2, int sel, int grid, cudaStream_t stream);
cudaError_t launch_bwd_prep(const BwdPrepParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_bwd_convert(const BwdConvertParams& p, int num_sms, cudaStream_t stream);

__host__ __device__ inline int bwd_units(int BH, int NK) { return BH * ((NK + kBwdBK - 1) / kBwdBK); }

// Work units of the forward: (bh, 128-row query tile) pairs, times the key splits.
__host__ __device__ inline int fwd_units(int BH, int NQ, int nsplit = 1) {
  return BH * ((NQ + kFwdBQ - 1) / kFwdBQ) * (nsplit > 1 ? nsplit : 1);
}

}  // namespace skl
