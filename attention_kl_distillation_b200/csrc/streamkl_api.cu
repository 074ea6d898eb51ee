// streamkl_api.cu -- the C ABI of libstreamkl (declared in include/streamkl.h).
//
// Host-side only: argument validation, device capability checks, TMA
// descriptor construction (cached per pointer and shape), and kernel launches
// on the caller's stream.  No device memory is allocated here; the backward's
// accumulator lives in a caller-provided workspace.
#include "streamkl.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>

#include "kernels.h"

namespace {

__device__ int g_device_status;  // set by kernels (atomicCAS from 0), read + cleared by the host

constexpr int kMaxDevices = 64;

std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_fault_mode{0};  // one-shot test hook, see streamkl_debug_inject

struct DeviceInfo {
  bool probed = false;
  bool sm100 = false;
  int num_sms = 0;
  int* status = nullptr;  // device address of g_device_status
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];
// Settings any host thread may change while others launch: atomics, written by
// the setters and initialised once from the environment on first read.
std::atomic<unsigned long long> g_wait_limit_ns{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

unsigned long long wait_limit_ns() {
  unsigned long long v = g_wait_limit_ns.load();
  if (v == 0) {
    long ms = 2000;
    if (const char* e = std::getenv("STREAMKL_WAIT_LIMIT_MS")) {
      long x = std::strtol(e, nullptr, 10);
      if (x >= 1) ms = x;
    }
    unsigned long long expect = 0;
    // a concurrent streamkl_set_wait_limit_ms wins over the environment default
    g_wait_limit_ns.compare_exchange_strong(expect, static_cast<unsigned long long>(ms) * 1000000ull);
    v = g_wait_limit_ns.load();
  }
  return v;
}

// Device of the current thread, probed once: sm_100 check, SM count, status word.
streamkl_status current_device(DeviceInfo** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return STREAMKL_ECUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.probed) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return STREAMKL_ECUDA;
    d.sm100 = (prop.major == 10 && prop.minor == 0);
    d.num_sms = prop.multiProcessorCount;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_status) != cudaSuccess) return STREAMKL_ECUDA;
    d.status = static_cast<int*>(addr);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return STREAMKL_ECUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    d.probed = true;
  }
  if (!d.sm100) return STREAMKL_EUNSUPPORTED;
  *out = &d;
  return STREAMKL_OK;
}

// ------------------------------------------------------------ TMA descriptors
struct MapKey {
  const void* ptr;
  int64_t BH, N;
  int d, rows;
  bool operator==(const MapKey& o) const {
    return ptr == o.ptr && BH == o.BH && N == o.N && d == o.d && rows == o.rows;
  }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};
constexpr int kMapCache = 64;
MapEntry g_maps[kMapCache];
int g_map_next = 0;

// 3-D map over a contiguous bf16 tensor [BH][N][d]: boxes of 64 elements of d
// (128 bytes, the 128B-swizzle span) by `rows` rows by one head.
streamkl_status tensor_map(const void* ptr, int64_t BH, int64_t N, int d, int rows,
                           CUtensorMap* out) {
  MapKey key{ptr, BH, N, d, rows};
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& e : g_maps)
    if (e.used && e.key == key) {
      *out = e.map;
      return STREAMKL_OK;
    }
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2,
                           static_cast<cuuint64_t>(N) * static_cast<cuuint64_t>(d) * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap m;
  CUresult r = g_encode(&m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return STREAMKL_ECUDA;
  MapEntry& e = g_maps[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCache;
  e.key = key;
  e.map = m;
  e.used = true;
  *out = m;
  return STREAMKL_OK;
}

// ------------------------------------------------------------ validation
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

streamkl_status check_problem(const streamkl_problem* pr) {
  if (!pr) return STREAMKL_EINVAL;
  if (pr->B < 1 || pr->H < 1 || pr->NQ < 1 || pr->NK < 1) return STREAMKL_EINVAL;
  if (pr->causal != 0 && pr->causal != 1) return STREAMKL_EINVAL;
  if (pr->causal && pr->NQ > pr->NK) return STREAMKL_EINVAL;
  if (!std::isfinite(pr->s1) || !std::isfinite(pr->s2)) return STREAMKL_EINVAL;
  // TMA coordinates are 32-bit signed; head count also indexes the grid.
  const int64_t BH = static_cast<int64_t>(pr->B) * pr->H;
  if (BH > (1 << 30) || pr->NQ > (1 << 30) || pr->NK > (1 << 30)) return STREAMKL_EINVAL;
  if (BH * static_cast<int64_t>((pr->NQ + 127) / 128) > (1ll << 31) - 1) return STREAMKL_EINVAL;
  if (!((pr->d1 == 64 || pr->d1 == 128) && (pr->d2 == 64 || pr->d2 == 128)))
    return STREAMKL_EUNSUPPORTED;
  return STREAMKL_OK;
}

float scale_or_default(float s, int d) {
  return s > 0.f ? s : 1.0f / std::sqrt(static_cast<float>(d));
}

constexpr float kLog2e = 1.4426950408889634f;

// Backward workspace: the fp32 accumulator of the reduced gradient ([BH][NQ][ld]
// dQ for key-tile units, [BH][NK][ld] dK for query-tile units; sized for the
// larger), then the per-row records [BH][NQpad][8] fp32, then two work-unit
// counters; each part starts on a 256-byte boundary.
struct BwdWorkspace {
  size_t dqacc_elems, rowrec_off, counter_off, total;
  int NQpad;
};

// Backward algorithm: process-wide setting, environment default read once.
std::atomic<int> g_bwd_algo{-1};

int bwd_algo_setting() {
  int v = g_bwd_algo.load();
  if (v < 0) {
    int a = STREAMKL_BWD_AUTO;
    if (const char* e = std::getenv("STREAMKL_BWD_ALGO")) {
      if (!std::strcmp(e, "fused")) a = STREAMKL_BWD_FUSED;
      else if (!std::strcmp(e, "split")) a = STREAMKL_BWD_SPLIT;
      else if (!std::strcmp(e, "fused_key_tiles")) a = STREAMKL_BWD_FUSED_KEY_TILES;
      else if (!std::strcmp(e, "fused_query_tiles")) a = STREAMKL_BWD_FUSED_QUERY_TILES;
      else if (!std::strcmp(e, "fused_sides")) a = STREAMKL_BWD_FUSED_SIDES;
    }
    int expect = -1;
    // a concurrent streamkl_set_bwd_algorithm wins over the environment default
    g_bwd_algo.compare_exchange_strong(expect, a);
    v = g_bwd_algo.load();
  }
  return v;
}

// AUTO: the page keeps the fused kernel while its atomic reductions stay cheap
// and switches to separate kernels when they contend.  On B200 the fused
// kernels measured faster at every size tested, in or beyond L2: B1 H32 N16384
// d128 causal (537 MB fp32 accumulator) fused query tiles 8.2-8.6 ms, fused
// key tiles 9.4-9.7, split 10.4-10.7; B1 H80 N65536 d128 causal (5 GiB
// accumulator) 357, 365 and 400 ms (bench.py --compare-bwd).  So AUTO is FUSED at every
// size; SPLIT stays available explicitly.

// SMs of the current device for scheduling decisions; 148 (B200) when no
// device can be queried, so that the decision is the same on a host without one.
int sms_or_default() {
  int dev = -1, n = 0;
  if (cudaGetDevice(&dev) == cudaSuccess &&
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
    return n;
  cudaGetLastError();
  return 148;
}

// Fused orientation: query-tile units (dQ on chip, dK reduced) when there are
// enough of them to fill the SMs twice over, else key-tile units (dK on chip,
// dQ reduced), which have more units when N_Q is small.
streamkl_bwd_algorithm fused_orientation(const streamkl_problem& pr) {
  const int64_t BH = static_cast<int64_t>(pr.B) * pr.H;
  const int64_t units_q = BH * ((pr.NQ + skl::kBwdQtRows - 1) / skl::kBwdQtRows);
  return units_q >= 2 * static_cast<int64_t>(sms_or_default()) ? STREAMKL_BWD_FUSED_QUERY_TILES
                                                               : STREAMKL_BWD_FUSED_KEY_TILES;
}

// The concrete algorithm: SPLIT, FUSED_KEY_TILES or FUSED_QUERY_TILES.
streamkl_bwd_algorithm resolve_bwd_algo(const streamkl_problem& pr) {
  const int a = bwd_algo_setting();
  if (a == STREAMKL_BWD_SPLIT || a == STREAMKL_BWD_FUSED_KEY_TILES ||
      a == STREAMKL_BWD_FUSED_QUERY_TILES || a == STREAMKL_BWD_FUSED_SIDES)
    return static_cast<streamkl_bwd_algorithm>(a);
  return fused_orientation(pr);  // FUSED and AUTO
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

BwdWorkspace bwd_workspace_layout(const streamkl_problem& pr) {
  BwdWorkspace w;
  const size_t BH = static_cast<size_t>(pr.B) * pr.H;
  w.NQpad = (pr.NQ + skl::kBwdBQ - 1) / skl::kBwdBQ * skl::kBwdBQ;
  w.dqacc_elems = BH * static_cast<size_t>(pr.NQ > pr.NK ? pr.NQ : pr.NK) *
                  static_cast<size_t>(pr.d1 + pr.d2);
  w.rowrec_off = round256(w.dqacc_elems * sizeof(float));
  const size_t rec = BH * static_cast<size_t>(w.NQpad) * skl::kRowRec * sizeof(float);
  w.counter_off = w.rowrec_off + rec;  // two work-unit counters follow the records
  w.total = w.rowrec_off + round256(rec + 2 * sizeof(int));
  return w;
}

}  // namespace

extern "C" {

int streamkl_abi_version(void) { return 1; }

uint64_t streamkl_launch_count(void) { return g_launches.load(); }

const char* streamkl_status_string(streamkl_status st) {
  switch (st) {
    case STREAMKL_OK: return "ok";
    case STREAMKL_EINVAL: return "invalid argument";
    case STREAMKL_EUNSUPPORTED: return "unsupported configuration or device";
    case STREAMKL_ECUDA: return "CUDA error";
    case STREAMKL_ETIMEOUT: return "kernel pipeline wait timed out";
    case STREAMKL_EDEVICE: return "device-side error";
  }
  return "unknown status";
}

streamkl_status streamkl_debug_inject(int mode) {
  if (mode != 0 && mode != 1) return STREAMKL_EINVAL;
  g_fault_mode.store(mode);
  return STREAMKL_OK;
}

streamkl_status streamkl_set_bwd_algorithm(streamkl_bwd_algorithm algo) {
  if (algo != STREAMKL_BWD_AUTO && algo != STREAMKL_BWD_FUSED && algo != STREAMKL_BWD_SPLIT &&
      algo != STREAMKL_BWD_FUSED_KEY_TILES && algo != STREAMKL_BWD_FUSED_QUERY_TILES &&
      algo != STREAMKL_BWD_FUSED_SIDES)
    return STREAMKL_EINVAL;
  g_bwd_algo.store(algo);
  return STREAMKL_OK;
}

streamkl_bwd_algorithm streamkl_bwd_algorithm_for(const streamkl_problem* prob) {
  if (check_problem(prob) != STREAMKL_OK) return STREAMKL_BWD_AUTO;
  return resolve_bwd_algo(*prob);
}

streamkl_status streamkl_set_wait_limit_ms(int ms) {
  if (ms < 1) return STREAMKL_EINVAL;
  g_wait_limit_ns.store(static_cast<unsigned long long>(ms) * 1000000ull);
  return STREAMKL_OK;
}

streamkl_status streamkl_query_device_status(streamkl_stream_t stream) {
  DeviceInfo* dev = nullptr;
  streamkl_status st = current_device(&dev);
  if (st != STREAMKL_OK) return st;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STREAMKL_ECUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof v) != cudaSuccess) return STREAMKL_ECUDA;
  if (v != 0) {
    int zero = 0;
    if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof zero) != cudaSuccess)
      return STREAMKL_ECUDA;
  }
  if (v == 0) return STREAMKL_OK;
  if (v == STREAMKL_ETIMEOUT) return STREAMKL_ETIMEOUT;
  return STREAMKL_EDEVICE;
}

}  // extern "C"

namespace {

// Validates forward arguments and fills the parameter block (maps, outputs,
// scales, status word).  Split-K fields are left off.
streamkl_status prepare_fwd(const streamkl_problem* prob, const void* Q1, const void* K1,
                            const void* Q2, const void* K2, float* L, float* LSE1, float* LSE2,
                            skl::FwdParams* p, DeviceInfo** devp) {
  streamkl_status st = check_problem(prob);
  if (st != STREAMKL_OK) return st;
  const void* ins[4] = {Q1, K1, Q2, K2};
  for (const void* q : ins)
    if (!q || !aligned16(q)) return STREAMKL_EINVAL;
  if (!L || !LSE1 || !LSE2) return STREAMKL_EINVAL;
  if ((reinterpret_cast<uintptr_t>(L) | reinterpret_cast<uintptr_t>(LSE1) |
       reinterpret_cast<uintptr_t>(LSE2)) & 3u)
    return STREAMKL_EINVAL;
  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != STREAMKL_OK) return st;
  const int64_t BH = static_cast<int64_t>(prob->B) * prob->H;
  if ((st = tensor_map(K1, BH, prob->NK, prob->d1, skl::kFwdBK, &p->tmK1)) != STREAMKL_OK) return st;
  if ((st = tensor_map(K2, BH, prob->NK, prob->d2, skl::kFwdBK, &p->tmK2)) != STREAMKL_OK) return st;
  // Q tiles are TMA boxes: a query group of the transposed kernel, or the 128
  // rows of a row-tile unit (staged in shared memory, then copied into TMEM).
  const int qrows = prob->NQ <= skl::kFwdTMaxNQ ? skl::fwd_t_rows(prob->NQ) : skl::kFwdBQ;
  if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, qrows, &p->tmQ1)) != STREAMKL_OK) return st;
  if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, qrows, &p->tmQ2)) != STREAMKL_OK) return st;
  p->Q1 = static_cast<const __nv_bfloat16*>(Q1);
  p->Q2 = static_cast<const __nv_bfloat16*>(Q2);
  p->L = L;
  p->LSE1 = LSE1;
  p->LSE2 = LSE2;
  p->BH = static_cast<int>(BH);
  p->NQ = prob->NQ;
  p->NK = prob->NK;
  p->causal = prob->causal;
  p->c1 = scale_or_default(prob->s1, prob->d1) * kLog2e;
  p->c2 = scale_or_default(prob->s2, prob->d2) * kLog2e;
  p->status = dev->status;
  p->wait_limit_ns = wait_limit_ns();
  p->withhold_keys = g_fault_mode.exchange(0) == 1 ? 1 : 0;
  p->kt_chunk = 0;
  p->nsplit = 1;
  p->part = nullptr;
  // One head at a time once a head has a query tile per SM: the concurrent CTAs
  // then share its key tiles in L2 (B1 H32 N65536 causal: 52 -> 42 ms); smaller
  // problems keep the order that interleaves all heads per query tile, whose
  // last wave is shorter (N4096: 0.21 ms against 0.23).
  const int nqt = (prob->NQ + skl::kFwdBQ - 1) / skl::kFwdBQ;
  p->head_group = nqt >= dev->num_sms ? 1 : static_cast<int>(BH);
  *devp = dev;
  return STREAMKL_OK;
}

int fwd_key_tiles(const streamkl_problem& pr) { return (pr.NK + skl::kFwdBK - 1) / skl::kFwdBK; }

// The forward kernel for a problem: few query rows go to the transposed
// kernel (keys on the UMMA M axis), the rest to the 128-row tile kernel.
bool fwd_transposed(const streamkl_problem& pr) { return pr.NQ <= skl::kFwdTMaxNQ; }

// Forward work units, in 64 bits: the kernels count units in int, so a launch
// whose count does not fit is refused (EINVAL) before it is made.
int64_t fwd_unit_count64(const streamkl_problem& pr, int nsplit) {
  const int64_t BH = static_cast<int64_t>(pr.B) * pr.H;
  const int rows = fwd_transposed(pr) ? skl::fwd_t_rows(pr.NQ) : skl::kFwdBQ;
  return BH * ((pr.NQ + rows - 1) / rows) * (nsplit > 1 ? nsplit : 1);
}

int fwd_unit_count(const streamkl_problem& pr, int nsplit) {
  return static_cast<int>(fwd_unit_count64(pr, nsplit));
}

cudaError_t launch_fwd_any(const streamkl_problem& pr, const skl::FwdParams& p, int grid,
                           cudaStream_t s) {
  if (fwd_transposed(pr)) return skl::launch_fwd_t(p, pr.d1, pr.d2, skl::fwd_t_rows(pr.NQ), grid, s);
  return skl::launch_fwd(p, pr.d1, pr.d2, grid, s);
}

// Key tiles per chunk and the effective chunk count for a requested split.
void split_shape(const streamkl_problem& pr, int nsplit, int* kt_chunk, int* nsp) {
  const int nkt = fwd_key_tiles(pr);
  if (nsplit > nkt) nsplit = nkt;
  if (nsplit < 1) nsplit = 1;
  const int chunk = (nkt + nsplit - 1) / nsplit;
  *kt_chunk = chunk;
  *nsp = (nkt + chunk - 1) / chunk;
}

}  // namespace

extern "C" {

streamkl_status streamkl_fwd(const streamkl_problem* prob, const void* Q1, const void* K1,
                             const void* Q2, const void* K2, float* L, float* LSE1, float* LSE2,
                             streamkl_stream_t stream) {
  skl::FwdParams p;
  DeviceInfo* dev = nullptr;
  streamkl_status st = prepare_fwd(prob, Q1, K1, Q2, K2, L, LSE1, LSE2, &p, &dev);
  if (st != STREAMKL_OK) return st;
  if (fwd_unit_count64(*prob, 1) > INT32_MAX) return STREAMKL_EINVAL;
  const int units = fwd_unit_count(*prob, 1);
  const int grid = units < dev->num_sms ? units : dev->num_sms;
  if (launch_fwd_any(*prob, p, grid, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return STREAMKL_ECUDA;
  g_launches.fetch_add(1);
  return STREAMKL_OK;
}

size_t streamkl_fwd_splitk_workspace_size(const streamkl_problem* prob, int nsplit) {
  if (check_problem(prob) != STREAMKL_OK || nsplit < 1) return 0;
  int chunk, nsp;
  split_shape(*prob, nsplit, &chunk, &nsp);
  const size_t rows = static_cast<size_t>(prob->B) * prob->H * static_cast<size_t>(prob->NQ);
  return round256(static_cast<size_t>(nsp) * 5 * rows * sizeof(float));
}

int streamkl_fwd_splitk_suggest(const streamkl_problem* prob) {
  if (check_problem(prob) != STREAMKL_OK) return 0;
  DeviceInfo* dev = nullptr;
  if (current_device(&dev) != STREAMKL_OK) return 0;
  const int units = fwd_unit_count(*prob, 1);
  const int sms = dev->num_sms;
  if (units >= sms) {
    // Enough units already; without the causal mask they are all the same
    // length, so a partly filled last wave idles SMs: split in two to four
    // chunks when that fills the waves clearly better (B2 H16 NQ=2048
    // NK=32768: 512 units are 3.46 waves, two chunks make 6.92).
    if (prob->causal) return 1;
    auto fill = [&](long long total) {
      const long long waves = (total + sms - 1) / sms;
      return static_cast<double>(total) / static_cast<double>(waves * sms);
    };
    int best = 1;
    double best_fill = fill(units);
    const int nkt = fwd_key_tiles(*prob);
    for (int n = 2; n <= 4 && n <= nkt; ++n) {
      int chunk, nsp;
      split_shape(*prob, n, &chunk, &nsp);
      const double f = fill(static_cast<long long>(units) * nsp);
      if (f > best_fill + 0.05) {
        best_fill = f;
        best = nsp;
      }
    }
    return best;
  }
  // About four units per SM: measured on B200 for B1 H32 NK=32768 (32 and 64
  // unsplit units), fewer splits leave HBM idle in the last waves and more add
  // per-unit work (Q load, lane merge) and merge traffic.
  int n = (4 * sms) / units;
  const int nkt = fwd_key_tiles(*prob);
  if (n > nkt) n = nkt;
  int chunk, best;
  split_shape(*prob, n < 1 ? 1 : n, &chunk, &best);
  return best < 1 ? 1 : best;
}

streamkl_status streamkl_fwd_splitk(const streamkl_problem* prob, const void* Q1, const void* K1,
                                    const void* Q2, const void* K2, float* L, float* LSE1,
                                    float* LSE2, int nsplit, void* workspace, size_t ws_bytes,
                                    streamkl_stream_t stream) {
  if (nsplit < 1) return STREAMKL_EINVAL;
  const size_t need = streamkl_fwd_splitk_workspace_size(prob, nsplit);
  if (need == 0) return check_problem(prob) != STREAMKL_OK ? check_problem(prob) : STREAMKL_EINVAL;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < need)
    return STREAMKL_EINVAL;
  skl::FwdParams p;
  DeviceInfo* dev = nullptr;
  streamkl_status st = prepare_fwd(prob, Q1, K1, Q2, K2, L, LSE1, LSE2, &p, &dev);
  if (st != STREAMKL_OK) return st;
  int chunk, nsp;
  split_shape(*prob, nsplit, &chunk, &nsp);
  if (fwd_unit_count64(*prob, nsp) > INT32_MAX) return STREAMKL_EINVAL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (nsp > 1) {
    p.kt_chunk = chunk;
    p.nsplit = nsp;
    p.part = static_cast<float*>(workspace);
  }
  const int units = fwd_unit_count(*prob, p.nsplit);
  const int grid = units < dev->num_sms ? units : dev->num_sms;
  if (launch_fwd_any(*prob, p, grid, s) != cudaSuccess) return STREAMKL_ECUDA;
  g_launches.fetch_add(1);
  if (nsp > 1) {
    skl::FwdMergeParams mp;
    mp.part = p.part;
    mp.L = L;
    mp.LSE1 = LSE1;
    mp.LSE2 = LSE2;
    mp.BH = p.BH;
    mp.NQ = p.NQ;
    mp.NK = p.NK;
    mp.causal = p.causal;
    mp.nsplit = nsp;
    mp.kt_chunk = chunk;
    if (skl::launch_fwd_merge(mp, dev->num_sms, s) != cudaSuccess) return STREAMKL_ECUDA;
    g_launches.fetch_add(1);
  }
  return STREAMKL_OK;
}

size_t streamkl_bwd_workspace_size(const streamkl_problem* prob) {
  if (check_problem(prob) != STREAMKL_OK) return 0;
  return bwd_workspace_layout(*prob).total;
}

streamkl_status streamkl_bwd(const streamkl_problem* prob, const float* dL, const void* Q1,
                             const void* K1, const void* Q2, const void* K2, const float* L,
                             const float* LSE1, const float* LSE2, void* dQ1, void* dK1, void* dQ2,
                             void* dK2, void* workspace, size_t ws_bytes,
                             streamkl_stream_t stream) {
  streamkl_status st = check_problem(prob);
  if (st != STREAMKL_OK) return st;
  const void* ins[4] = {Q1, K1, Q2, K2};
  for (const void* p : ins)
    if (!p || !aligned16(p)) return STREAMKL_EINVAL;
  const float* vecs[4] = {dL, L, LSE1, LSE2};
  for (const float* v : vecs)
    if (!v || (reinterpret_cast<uintptr_t>(v) & 3u)) return STREAMKL_EINVAL;
  void* outs[4] = {dQ1, dK1, dQ2, dK2};
  bool any = false;
  for (void* o : outs) {
    if (o && !aligned16(o)) return STREAMKL_EINVAL;
    any = any || o != nullptr;
  }
  if (!any) return STREAMKL_EINVAL;
  const BwdWorkspace lay = bwd_workspace_layout(*prob);
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) || ws_bytes < lay.total)
    return STREAMKL_EINVAL;

  DeviceInfo* dev = nullptr;
  if ((st = current_device(&dev)) != STREAMKL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  const int64_t BH = static_cast<int64_t>(prob->B) * prob->H;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* dqacc = reinterpret_cast<float*>(ws);
  float* rowrec = reinterpret_cast<float*>(ws + lay.rowrec_off);
  const float s1 = scale_or_default(prob->s1, prob->d1);
  const float s2 = scale_or_default(prob->s2, prob->d2);
  // Gradient sides asked for (the page's configurations).
  const int sel = ((dQ1 || dK1) ? 1 : 0) | ((dQ2 || dK2) ? 2 : 0);
  streamkl_bwd_algorithm algo = resolve_bwd_algo(*prob);
  // AUTO and FUSED run one side alone with 128-key steps when only one side is
  // asked for (B1 H32 N16384 d128 causal: student side 4.89 against 6.14 ms for
  // the query-tile kernel's one-sided instance, teacher side 4.90 against 6.30);
  // an explicit setting is kept.
  const int setting = bwd_algo_setting();
  if (algo == STREAMKL_BWD_FUSED_QUERY_TILES && sel != 3 &&
      (setting == STREAMKL_BWD_AUTO || setting == STREAMKL_BWD_FUSED))
    algo = STREAMKL_BWD_FUSED_SIDES;
  const bool split = algo == STREAMKL_BWD_SPLIT;
  const bool sides = algo == STREAMKL_BWD_FUSED_SIDES;
  const bool qtiles = algo == STREAMKL_BWD_FUSED_QUERY_TILES || sides;
  // the fused kernels accumulate one gradient in fp32: dQ over key tiles, dK over query tiles
  const bool want_acc = !split && (qtiles ? (dK1 || dK2) : (dQ1 || dQ2));
  // The fused kernels are specialised on the sides asked for, and their
  // accumulator holds only those sides' columns.
  const int ld1 = (sel & 1) ? prob->d1 : 0, ld2 = (sel & 2) ? prob->d2 : 0;
  int* counters = reinterpret_cast<int*>(ws + lay.counter_off);

  skl::BwdPrepParams pp;
  pp.L = L;
  pp.LSE1 = LSE1;
  pp.LSE2 = LSE2;
  pp.dL = dL;
  pp.rowrec = qtiles ? nullptr : rowrec;  // the query-tile kernel reads L, LSE and dL itself
  pp.dQacc = dqacc;
  pp.dqacc_elems = want_acc ? BH * static_cast<int64_t>(qtiles ? prob->NK : prob->NQ) * (ld1 + ld2) : 0;
  pp.counters = counters;
  pp.BH = static_cast<int>(BH);
  pp.NQ = prob->NQ;
  pp.NQpad = lay.NQpad;
  pp.s1 = s1;
  pp.s2 = s2;
  if (skl::launch_bwd_prep(pp, dev->num_sms, s) != cudaSuccess) return STREAMKL_ECUDA;
  g_launches.fetch_add(1);

  if (split) {
    skl::BwdSplitParams sp;
    sp.rowrec = rowrec;
    sp.BH = static_cast<int>(BH);
    sp.NQ = prob->NQ;
    sp.NK = prob->NK;
    sp.NQpad = lay.NQpad;
    sp.causal = prob->causal;
    sp.c1 = s1 * kLog2e;
    sp.c2 = s2 * kLog2e;
    sp.status = dev->status;
    sp.wait_limit_ns = wait_limit_ns();
    if (dK1 || dK2) {  // dK pass: resident key tiles, streamed query tiles
      if ((st = tensor_map(K1, BH, prob->NK, prob->d1, 128, &sp.tmR1)) != STREAMKL_OK) return st;
      if ((st = tensor_map(K2, BH, prob->NK, prob->d2, 128, &sp.tmR2)) != STREAMKL_OK) return st;
      if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, 64, &sp.tmC1)) != STREAMKL_OK) return st;
      if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, 64, &sp.tmC2)) != STREAMKL_OK) return st;
      sp.counter = counters;
      sp.out1 = static_cast<__nv_bfloat16*>(dK1);
      sp.out2 = static_cast<__nv_bfloat16*>(dK2);
      const int units = static_cast<int>(BH) * ((prob->NK + 127) / 128);
      if (skl::launch_bwd_split(sp, skl::BwdPass::kDK, prob->d1, prob->d2,
                                units < dev->num_sms ? units : dev->num_sms, s) != cudaSuccess)
        return STREAMKL_ECUDA;
      g_launches.fetch_add(1);
    }
    if (dQ1 || dQ2) {  // dQ pass: resident query tiles, streamed key tiles
      if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, 128, &sp.tmR1)) != STREAMKL_OK) return st;
      if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, 128, &sp.tmR2)) != STREAMKL_OK) return st;
      if ((st = tensor_map(K1, BH, prob->NK, prob->d1, 64, &sp.tmC1)) != STREAMKL_OK) return st;
      if ((st = tensor_map(K2, BH, prob->NK, prob->d2, 64, &sp.tmC2)) != STREAMKL_OK) return st;
      sp.counter = counters + 1;
      sp.out1 = static_cast<__nv_bfloat16*>(dQ1);
      sp.out2 = static_cast<__nv_bfloat16*>(dQ2);
      const int units = static_cast<int>(BH) * ((prob->NQ + 127) / 128);
      if (skl::launch_bwd_split(sp, skl::BwdPass::kDQ, prob->d1, prob->d2,
                                units < dev->num_sms ? units : dev->num_sms, s) != cudaSuccess)
        return STREAMKL_ECUDA;
      g_launches.fetch_add(1);
    }
    return STREAMKL_OK;
  }

  if (sides) {
    skl::BwdSideParams p;
    if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, 128, &p.tmQ1)) != STREAMKL_OK) return st;
    if ((st = tensor_map(K1, BH, prob->NK, prob->d1, 128, &p.tmK1)) != STREAMKL_OK) return st;
    if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, 128, &p.tmQ2)) != STREAMKL_OK) return st;
    if ((st = tensor_map(K2, BH, prob->NK, prob->d2, 128, &p.tmK2)) != STREAMKL_OK) return st;
    p.L = L;
    p.LSE1 = LSE1;
    p.LSE2 = LSE2;
    p.dL = dL;
    p.dKacc = dqacc;
    p.ldk = ld1 + ld2;
    p.BH = static_cast<int>(BH);
    p.NQ = prob->NQ;
    p.NK = prob->NK;
    p.causal = prob->causal;
    p.c1 = s1 * kLog2e;
    p.c2 = s2 * kLog2e;
    p.s1 = s1;
    p.s2 = s2;
    p.status = dev->status;
    p.wait_limit_ns = wait_limit_ns();
    const int units = skl::bwd_qt_units(p.BH, p.NQ);
    const int grid = units < dev->num_sms ? units : dev->num_sms;
    for (int side = 1; side <= 2; ++side) {
      if (!(sel & side)) continue;
      p.dQ = static_cast<__nv_bfloat16*>(side == 1 ? dQ1 : dQ2);
      p.want_dq = p.dQ != nullptr;
      p.want_dk = (side == 1 ? dK1 : dK2) != nullptr;
      p.dk_col = side == 1 ? 0 : ld1;
      p.counter = counters + (side - 1);
      if (skl::launch_bwd_side(p, prob->d1, prob->d2, side, grid, s) != cudaSuccess)
        return STREAMKL_ECUDA;
      g_launches.fetch_add(1);
    }
    if (want_acc) {
      skl::BwdConvertParams cp;
      cp.dQacc = dqacc;
      cp.dQ1 = static_cast<__nv_bfloat16*>(dK1);
      cp.dQ2 = static_cast<__nv_bfloat16*>(dK2);
      cp.rows = BH * prob->NK;
      cp.d1 = ld1;
      cp.d2 = ld2;
      if (skl::launch_bwd_convert(cp, dev->num_sms, s) != cudaSuccess) return STREAMKL_ECUDA;
      g_launches.fetch_add(1);
    }
    return STREAMKL_OK;
  }

  if (qtiles) {
    skl::BwdQtParams p;
    if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, skl::kBwdQtRows, &p.tmQ1)) != STREAMKL_OK) return st;
    if ((st = tensor_map(K1, BH, prob->NK, prob->d1, skl::kBwdQtKeys, &p.tmK1)) != STREAMKL_OK) return st;
    if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, skl::kBwdQtRows, &p.tmQ2)) != STREAMKL_OK) return st;
    if ((st = tensor_map(K2, BH, prob->NK, prob->d2, skl::kBwdQtKeys, &p.tmK2)) != STREAMKL_OK) return st;
    p.L = L;
    p.LSE1 = LSE1;
    p.LSE2 = LSE2;
    p.dL = dL;
    p.dKacc = dqacc;
    p.counter = counters;
    p.dQ1 = static_cast<__nv_bfloat16*>(dQ1);
    p.dQ2 = static_cast<__nv_bfloat16*>(dQ2);
    p.BH = static_cast<int>(BH);
    p.NQ = prob->NQ;
    p.NK = prob->NK;
    p.causal = prob->causal;
    p.want_dq1 = dQ1 != nullptr;
    p.want_dk1 = dK1 != nullptr;
    p.want_dq2 = dQ2 != nullptr;
    p.want_dk2 = dK2 != nullptr;
    p.c1 = s1 * kLog2e;
    p.c2 = s2 * kLog2e;
    p.s1 = s1;
    p.s2 = s2;
    p.status = dev->status;
    p.wait_limit_ns = wait_limit_ns();
    const int units = skl::bwd_qt_units(p.BH, p.NQ);
    const int grid = units < dev->num_sms ? units : dev->num_sms;
    if (skl::launch_bwd_qt(p, prob->d1, prob->d2, sel, grid, s) != cudaSuccess) return STREAMKL_ECUDA;
    g_launches.fetch_add(1);
    if (want_acc) {
      skl::BwdConvertParams cp;
      cp.dQacc = dqacc;
      cp.dQ1 = static_cast<__nv_bfloat16*>(dK1);
      cp.dQ2 = static_cast<__nv_bfloat16*>(dK2);
      cp.rows = BH * prob->NK;
      cp.d1 = ld1;  // accumulator columns: teacher side (if selected), then student side
      cp.d2 = ld2;
      if (skl::launch_bwd_convert(cp, dev->num_sms, s) != cudaSuccess) return STREAMKL_ECUDA;
      g_launches.fetch_add(1);
    }
    return STREAMKL_OK;
  }

  skl::BwdParams p;
  if ((st = tensor_map(Q1, BH, prob->NQ, prob->d1, skl::kBwdBQ, &p.tmQ1)) != STREAMKL_OK) return st;
  if ((st = tensor_map(K1, BH, prob->NK, prob->d1, skl::kBwdBK, &p.tmK1)) != STREAMKL_OK) return st;
  if ((st = tensor_map(Q2, BH, prob->NQ, prob->d2, skl::kBwdBQ, &p.tmQ2)) != STREAMKL_OK) return st;
  if ((st = tensor_map(K2, BH, prob->NK, prob->d2, skl::kBwdBK, &p.tmK2)) != STREAMKL_OK) return st;
  p.rowrec = rowrec;
  p.dQacc = dqacc;
  p.dK1 = static_cast<__nv_bfloat16*>(dK1);
  p.dK2 = static_cast<__nv_bfloat16*>(dK2);
  p.BH = static_cast<int>(BH);
  p.NQ = prob->NQ;
  p.NK = prob->NK;
  p.NQpad = lay.NQpad;
  p.causal = prob->causal;
  p.want_dq1 = dQ1 != nullptr;
  p.want_dk1 = dK1 != nullptr;
  p.want_dq2 = dQ2 != nullptr;
  p.want_dk2 = dK2 != nullptr;
  p.c1 = s1 * kLog2e;
  p.c2 = s2 * kLog2e;
  p.status = dev->status;
  p.wait_limit_ns = wait_limit_ns();
  const int units = skl::bwd_units(p.BH, p.NK);
  const int grid = units < dev->num_sms ? units : dev->num_sms;
  if (skl::launch_bwd(p, prob->d1, prob->d2, sel, grid, s) != cudaSuccess) return STREAMKL_ECUDA;
  g_launches.fetch_add(1);

  if (want_acc) {
    skl::BwdConvertParams cp;
    cp.dQacc = dqacc;
    cp.dQ1 = static_cast<__nv_bfloat16*>(dQ1);
    cp.dQ2 = static_cast<__nv_bfloat16*>(dQ2);
    cp.rows = BH * prob->NQ;
    cp.d1 = ld1;  // accumulator columns: teacher side (if selected), then student side
    cp.d2 = ld2;
    if (skl::launch_bwd_convert(cp, dev->num_sms, s) != cudaSuccess) return STREAMKL_ECUDA;
    g_launches.fetch_add(1);
  }
  return STREAMKL_OK;
}

}  // extern "C"
