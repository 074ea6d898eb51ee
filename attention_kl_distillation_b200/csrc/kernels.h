// kernels.h -- parameter blocks and launchers shared between the C-ABI layer
// (streamkl_api.cu) and the sm_100a kernels.  Internal to libstreamkl.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace skl {

// Rows of Q in one forward tile (the UMMA M dimension and the TMEM lanes).
constexpr int kFwdBQ = 128;
// Keys per forward tile (UMMA N).
constexpr int kFwdBK = 64;

struct FwdParams {
  CUtensorMap tmQ1, tmK1, tmQ2, tmK2;  // 3-D maps over [BH][N][d], 128B swizzle
  float* L;
  float* LSE1;
  float* LSE2;
  int BH, NQ, NK, causal;
  float c1, c2;  // s_t * log2(e): logits in the base-2 domain
  int* status;   // device status word
  unsigned long long wait_limit_ns;
};

// Dynamic shared memory the forward kernel needs for head dims (d1, d2).
size_t fwd_smem_bytes(int d1, int d2);

// Launch the forward kernel; returns the launch error.
cudaError_t launch_fwd(const FwdParams& p, int d1, int d2, int grid, cudaStream_t stream);

// Work units of the forward: (bh, 128-row query tile) pairs.
__host__ __device__ inline int fwd_units(int BH, int NQ) { return BH * ((NQ + kFwdBQ - 1) / kFwdBQ); }

}  // namespace skl
