/*
 * streamkl.h -- C ABI of libstreamkl: fused single-pass attention KL
 * divergence on NVIDIA B200 (sm_100a).
 *
 * Operation (StreamKL summary page, "Metodologia", section 1 "Formulazione
 * Online"): for batch b, head h and query row i,
 *
 *   x1[i,j] = s1 * <Q1[i], K1[j]>,  x2[i,j] = s2 * <Q2[i], K2[j]>
 *   P_t[i,:] = softmax over the visible keys of x_t[i,:]
 *   LSE_t[i] = log sum_j exp(x_t[i,j])
 *   L[i]     = KL(P1[i,:] || P2[i,:]) = sum_j P1 * ((x1 - LSE1) - (x2 - LSE2))   (nats)
 *
 * computed in one pass over the keys without materialising the N_Q x N_K
 * maps.  The backward (section 2, "Strategia di Ricalcolo") regenerates the
 * probabilities tile by tile from the saved L, LSE1 and LSE2 and returns the
 * gradients of sum_i dL[i] * L[i] for both gradient configurations of the
 * page (teacher fixed: dQ2/dK2; student fixed: dQ1/dK1).
 *
 * Conventions shared by every entry point:
 *  - Tensors are device pointers, contiguous, row-major:
 *      Q1 [B][H][NQ][d1], K1 [B][H][NK][d1], Q2 [B][H][NQ][d2], K2 [B][H][NK][d2]
 *    in bf16 (IEEE binary32 with the low 16 bits dropped), 16-byte aligned.
 *  - Row vectors L, LSE1, LSE2, dL are fp32 [B][H][NQ].
 *  - Causal masking is bottom-right aligned: key j is visible from row i when
 *    j <= i + NK - NQ (the usual j <= i when NQ == NK).  Causal with NQ > NK
 *    is rejected, since some rows would see no key.
 *  - The caller owns every buffer.  The library allocates no device memory on
 *    any call below; host-side it keeps a small cache of TMA descriptors.
 *  - Calls are asynchronous on the given stream (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument errors are returned synchronously and
 *    launch nothing.  A kernel that detects a stalled pipeline records
 *    STREAMKL_ETIMEOUT in a device status word and exits;
 *    streamkl_query_device_status reads it.
 */
#ifndef STREAMKL_H_
#define STREAMKL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, declared here so the header needs no CUDA include. */
typedef struct CUstream_st *streamkl_stream_t;

typedef enum {
  STREAMKL_OK = 0,
  STREAMKL_EINVAL = 1,       /* bad argument: null/unaligned pointer, bad size, bad workspace */
  STREAMKL_EUNSUPPORTED = 2, /* valid but not built: head dims other than 64/128, no sm_100 device */
  STREAMKL_ECUDA = 3,        /* a CUDA runtime/driver call or a launch failed */
  STREAMKL_ETIMEOUT = 4,     /* a kernel gave up on a pipeline wait (device status word) */
  STREAMKL_EDEVICE = 5       /* any other error recorded by a kernel */
} streamkl_status;

/*
 * Problem description.  B, H, NQ, NK >= 1; d1, d2 in {64, 128}; causal 0/1.
 * s1, s2: softmax scales of the two distributions; a value <= 0 selects
 * 1/sqrt(d_t).  The two distributions may have different head dimensions
 * (teacher d1, student d2) but share B, H, NQ and NK.
 */
typedef struct {
  int B, H, NQ, NK, d1, d2, causal;
  float s1, s2;
} streamkl_problem;

/*
 * Forward: L, LSE1, LSE2 [B][H][NQ] fp32 from Q1, K1, Q2, K2 (bf16).
 * Section 1 of the page: the five running scalars m1, m2, l1, l2 and acc per
 * row, finished as L = acc/l1 + LSE2 - LSE1 with LSE_t = m_t + log l_t; key
 * tiles past the causal frontier are skipped.  L, LSE1 and LSE2 are also
 * the saved state of section 2 that streamkl_bwd consumes.  Problems with
 * NQ <= 32 run a transposed kernel (keys on the MMA's long axis, as in the
 * ETAP page's S^T = K Q^T); the results agree with the row-tile kernel to
 * fp32 rounding.
 * Errors: EINVAL (null or unaligned pointer, sizes out of range, causal with
 * NQ > NK), EUNSUPPORTED (d not in {64,128}, device is not sm_100), ECUDA.
 */
streamkl_status streamkl_fwd(const streamkl_problem *prob, const void *Q1, const void *K1,
                             const void *Q2, const void *K2, float *L, float *LSE1, float *LSE2,
                             streamkl_stream_t stream);

/*
 * Split-K forward (section 3, "Variante Split-K": for few query rows, e.g. a
 * decode step with N_Q = 1, the keys are partitioned across thread blocks so
 * that every SM has work).  Same results as streamkl_fwd within rounding.
 * The keys of every 128-row query tile are cut into `nsplit` chunks of equal
 * length (in 128-key tiles); each chunk's tiles write partial row states
 * (m1, m2, l1, l2, acc) to `workspace`, and a merge kernel combines them into
 * L, LSE1, LSE2.  nsplit >= 1 (1 = no split); nsplit above the number of key
 * tiles is clamped.  workspace: streamkl_fwd_splitk_workspace_size(prob,
 * nsplit) bytes of device memory, 256-byte aligned, caller-owned; contents on
 * entry do not matter.  Errors: as streamkl_fwd, plus EINVAL for nsplit < 1
 * or a short/unaligned workspace.
 */
streamkl_status streamkl_fwd_splitk(const streamkl_problem *prob, const void *Q1, const void *K1,
                                    const void *Q2, const void *K2, float *L, float *LSE1,
                                    float *LSE2, int nsplit, void *workspace, size_t ws_bytes,
                                    streamkl_stream_t stream);

/* Workspace bytes for streamkl_fwd_splitk (0 on a bad problem or nsplit < 1). */
size_t streamkl_fwd_splitk_workspace_size(const streamkl_problem *prob, int nsplit);

/*
 * A split count for the current device: about four of the forward's work
 * units per SM (at most one key tile per chunk).  When the problem already
 * has a unit per SM: 1 for a causal problem; otherwise the count from 1 to 4
 * that fills the last wave of SMs clearly best (all units have the same
 * length, so a partly filled last wave idles SMs).  0 on a bad problem or if
 * the device cannot be queried.
 */
int streamkl_fwd_splitk_suggest(const streamkl_problem *prob);

/*
 * Workspace bytes that streamkl_bwd needs for this problem: an fp32
 * accumulator for the gradient the fused kernels reduce across tiles (section
 * 2, "Fusione del Kernel": dQ with atomics across key tiles, or dK across
 * query tiles), [B][H][max(NQ,NK)][d1+d2], plus per-row records and padding.
 * The same size serves every algorithm.  0 on a bad problem.
 */
size_t streamkl_bwd_workspace_size(const streamkl_problem *prob);

/*
 * Backward: gradients of sum_i dL[i] * L[i] (section 2).  Inputs are the
 * forward inputs plus the saved L, LSE1, LSE2 from streamkl_fwd and the
 * upstream dL (fp32 [B][H][NQ]).  Outputs dQ1, dK1, dQ2, dK2 are bf16 with the
 * shapes of their inputs; any of them may be NULL, which skips it: dQ1 = dK1
 * = NULL is the page's configuration 1 (teacher P1 fixed), dQ2 = dK2 = NULL
 * its configuration 2 (student P2 fixed).  With one side asked for, the fused
 * algorithm runs a kernel specialised to it: only that side's dS is formed
 * and contracted (for the teacher side without the student's exponential).
 * workspace must hold
 * streamkl_bwd_workspace_size bytes of device memory, 256-byte aligned; its
 * contents on entry do not matter and on exit are unspecified.  Gradients are
 * not bitwise reproducible (fp32 atomics).
 * Errors: as streamkl_fwd, plus EINVAL for a short or unaligned workspace or
 * all four outputs NULL.
 */
streamkl_status streamkl_bwd(const streamkl_problem *prob, const float *dL, const void *Q1,
                             const void *K1, const void *Q2, const void *K2, const float *L,
                             const float *LSE1, const float *LSE2, void *dQ1, void *dK1, void *dQ2,
                             void *dK2, void *workspace, size_t ws_bytes, streamkl_stream_t stream);

/*
 * Device scratch owned by streamkl_bwd_noalloc: 64 MiB per GPU.  It is a
 * static device array of the library's module, so it is reserved on a GPU
 * when the module is loaded there and held until the process exits.  With
 * eager module loading that happens at context creation; under CUDA's lazy
 * loading (the default since CUDA 12.2, CUDA_MODULE_LOADING=LAZY) it happens
 * at the module's first use on that GPU, which is the first
 * streamkl_bwd_noalloc call (its address lookup) or the first launch of any
 * of the library's kernels there.
 */
#define STREAMKL_NOALLOC_SCRATCH_BYTES (64u << 20)

/* STREAMKL_NOALLOC_SCRATCH_BYTES as the built library has it (no CUDA call). */
size_t streamkl_bwd_noalloc_scratch_bytes(void);

/*
 * Backward for callers that cannot allocate device memory (the paper has no
 * counterpart; it is an interface convenience).  Such callers include a
 * framework whose caching allocator already holds the free device memory, or
 * code that must not call cudaMalloc/cudaFree because those may synchronise
 * the device.  Same arguments, results and errors as streamkl_bwd, without
 * the workspace: the library uses its own static device scratch instead and
 * calls no cudaMalloc, cudaFree or other allocating routine.
 *  - Problems whose streamkl_bwd_workspace_size exceeds
 *    STREAMKL_NOALLOC_SCRATCH_BYTES are rejected with STREAMKL_EINVAL before
 *    any CUDA call.
 *  - The first call on a device looks up the scratch's device address
 *    (cudaGetSymbolAddress) with that device current; under lazy module
 *    loading that lookup is also what loads the module and reserves the
 *    scratch on that device.  Make that first call before any stream
 *    capture.
 *  - Every call on a device shares the one scratch array, which keeps the
 *    last call's contents (each call clears what must start at zero).  Calls
 *    that overlap on the GPU (different streams, or threads without ordering)
 *    race on it and give wrong gradients: order them on one stream.
 */
streamkl_status streamkl_bwd_noalloc(const streamkl_problem *prob, const float *dL,
                                     const void *Q1, const void *K1, const void *Q2,
                                     const void *K2, const float *L, const float *LSE1,
                                     const float *LSE2, void *dQ1, void *dK1, void *dQ2,
                                     void *dK2, streamkl_stream_t stream);

/*
 * How streamkl_bwd computes the gradients (section 2, "Fusione del Kernel",
 * and the fused-versus-separate ablation):
 *  FUSED_KEY_TILES    one kernel visits every (query tile, key tile) pair
 *                     once, with 128-key work units; dK stays on chip, dQ is
 *                     accumulated across key tiles with fp32 reductions into
 *                     the workspace (the page's design), then converted.
 *  FUSED_QUERY_TILES  the same with 128-query work units: dQ stays on chip and
 *                     dK is accumulated across query tiles with fp32
 *                     reductions.  Each dS thread then owns a query row, so
 *                     its L, LSE and dL are registers instead of shared-memory
 *                     loads for every key.
 *  FUSED_SIDES        query-tile units with one gradient side per pass and
 *                     128-key steps: every product is N = 128, both S
 *                     products are recomputed once per side asked for.
 *  FUSED              the fused orientation chosen by shape: query tiles when
 *                     B*H*ceil(NQ/128) fills the device's SMs twice, else key
 *                     tiles; with query tiles and one side asked for,
 *                     FUSED_SIDES (measured faster for one side).
 *  SPLIT              two passes of one kernel: a dK pass over key tiles and
 *                     a dQ pass over query tiles, each regenerating the
 *                     probabilities; no reductions in global memory.
 *  AUTO               FUSED.  The page switches to separate kernels when the
 *                     atomics contend; on B200 the fused kernels measured
 *                     faster at every size tested, up to a 5 GiB fp32
 *                     accumulator (B1 H80 N65536 d128 causal: fused 357 ms,
 *                     split 400 ms), so AUTO does not pick SPLIT.
 * Results agree within rounding either way.  Process-wide; default AUTO (or
 * the environment variable STREAMKL_BWD_ALGO = auto | fused | split |
 * fused_key_tiles | fused_query_tiles, read once).
 */
typedef enum {
  STREAMKL_BWD_AUTO = 0,
  STREAMKL_BWD_FUSED = 1,
  STREAMKL_BWD_SPLIT = 2,
  STREAMKL_BWD_FUSED_KEY_TILES = 3,
  STREAMKL_BWD_FUSED_QUERY_TILES = 4,
  STREAMKL_BWD_FUSED_SIDES = 5
} streamkl_bwd_algorithm;

streamkl_status streamkl_set_bwd_algorithm(streamkl_bwd_algorithm algo);

/* The algorithm streamkl_bwd would use for this problem on the current device
 * when both sides are asked for: SPLIT, FUSED_KEY_TILES, FUSED_QUERY_TILES or
 * FUSED_SIDES (AUTO and FUSED resolved; for one side, FUSED_QUERY_TILES under
 * AUTO or FUSED runs as FUSED_SIDES). */
streamkl_bwd_algorithm streamkl_bwd_algorithm_for(const streamkl_problem *prob);

/* Static English text for a status code. */
const char *streamkl_status_string(streamkl_status st);

/*
 * Synchronises `stream`, then reads and clears the device status word that
 * kernels set when a pipeline wait times out.  Returns STREAMKL_OK when no
 * kernel has recorded an error since the last call, else the recorded code.
 */
streamkl_status streamkl_query_device_status(streamkl_stream_t stream);

/*
 * Upper bound, in milliseconds, on any single wait inside a kernel before it
 * gives up with STREAMKL_ETIMEOUT (default 2000; also read once from the
 * environment variable STREAMKL_WAIT_LIMIT_MS).  Values < 1 are rejected.
 */
streamkl_status streamkl_set_wait_limit_ms(int ms);

/*
 * Test hook for failure detection (no counterpart on the page).  mode 1 arms a
 * one-shot fault: in the next streamkl_fwd launch the TMA producer issues no
 * key tiles, so the UMMA warp's wait for them runs past the wait limit.  The
 * kernel then records STREAMKL_ETIMEOUT, every role of every CTA unwinds (in-
 * flight copies land, TMEM is freed) and the launch ends; the CUDA context
 * stays usable.  mode 0 disarms.  Nothing faults, traps or hangs.
 */
streamkl_status streamkl_debug_inject(int mode);

/* Version of this ABI: 1. */
int streamkl_abi_version(void);

/*
 * Number of kernels this library has launched successfully in this process
 * (all devices, all entry points).  Lets a caller count the device work a
 * sequence of calls issued.
 */
uint64_t streamkl_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMKL_H_ */
