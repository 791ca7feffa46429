/*
 * fa.h -- C ABI of libfa: exact scaled dot-product attention on one B200
 * (sm_100a), forward and backward.
 *
 * The operation ("NVIDIA Blackwell: FlashAttention-4 Overcomes Memory
 * Bottlenecks", body; "NVIDIA's FlashAttention-4: Cementing AI Infrastructure
 * Dominance", "The Technical Edge"): for every (batch b, head h)
 *
 *     S    = scale * Q K^T,  with keys j > i masked out when causal
 *            (queries and keys aligned at position 0)
 *     LSE  = natural-log log-sum-exp of each row of S
 *     O    = softmax(S) V = exp(S - LSE) V
 *
 * and the backward pass (recomputing P = exp(S - LSE) from the saved LSE):
 *
 *     dV = P^T dO,  dP = dO V^T,  D = rowsum(dO * O),  dS = P * (dP - D),
 *     dQ = scale * dS K,  dK = scale * dS^T Q.
 *
 * Layout: every tensor is contiguous [B, H, N, d] (d fastest), bf16 for
 * Q, K, V, O, dO, dQ, dK, dV and fp32 for LSE ([B, H, N]).  All data
 * pointers are DEVICE pointers; the caller owns every buffer.  The library
 * allocates no device memory on any call; it keeps only a per-device status
 * word and cached kernel attributes.
 *
 * Calls are asynchronous on the caller's stream (`stream` is a cudaStream_t,
 * NULL = legacy default stream).  Argument checks happen on the host before
 * anything is launched; a failing check returns its code and launches
 * nothing.  No C++ exception crosses this interface and nothing calls exit.
 *
 * Supported: d in {64, 128}; any N >= 1 (a ragged last tile is masked);
 * 0 < scale < inf.  Every pointer must be 16-byte aligned (TMA), and outputs
 * must not overlap inputs.  Results are deterministic except dQ, whose fp32
 * accumulation order (atomic adds across key tiles) varies between runs at
 * the level of fp32 rounding.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad flag, bad scale, overlap */
  FA_ERR_UNSUPPORTED = 2, /* head dim other than 64/128, sizes beyond the index range */
  FA_ERR_ALIGNMENT = 3,   /* a pointer not 16-byte aligned */
  FA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed (launch, attributes, TMA encode) */
  FA_ERR_TIMEOUT = 5      /* a kernel's bounded pipeline wait expired (see fa_last_device_status) */
} fa_status;

/*
 * Forward.  Q, K, V: bf16 [B, H, N, d] (read).  O: bf16 [B, H, N, d]
 * (written).  LSE: fp32 [B, H, N] (written), natural log: LSE_i =
 * ln sum_j exp(S_ij).  B, H or N equal to 0 is an empty problem: returns
 * FA_OK and launches nothing.  causal: 0 or 1.
 * One kernel launch on `stream`.
 */
int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
           float scale, int causal, void* stream);

/*
 * Bytes of device workspace fa_bwd needs: an fp32 dQ accumulator
 * [B, H, Npad, d] plus fp32 D and LSE*log2(e) vectors [B, H, Npad], with
 * Npad = N rounded up to a multiple of 128, each part 256-byte aligned.
 * Returns 0 for an empty or invalid shape.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward.  Q, K, V, O, dO: bf16 [B, H, N, d] (read); LSE: fp32 [B, H, N]
 * as written by fa_fwd for the same Q, K, V, scale and causal (read).
 * dQ, dK, dV: bf16 [B, H, N, d] (written).  workspace: device memory of at
 * least fa_bwd_workspace_size() bytes, 16-byte aligned, owned by the caller;
 * its contents on entry do not matter and it may be reused after the call's
 * work on `stream` has finished.  Three kernel launches on `stream`
 * (preprocess, main, dQ conversion).  Two fa_bwd calls that share a
 * workspace must not overlap in time.
 */
int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
           void* dQ, void* dK, void* dV, void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
           float scale, int causal, void* stream);

/*
 * Grouped-query attention and unequal query / key lengths (prefill of new
 * queries against a cache of earlier keys, the serving use the pages name for
 * FlashAttention-4 -- "NVIDIA Blackwell: FlashAttention-4 Overcomes Memory
 * Bottlenecks", body, on SGLang / vLLM prefill; GQA / MQA support is listed
 * as missing in "NVIDIA's FlashAttention-4: Cementing AI Infrastructure
 * Dominance in 2025", "Limitations and the Road Ahead").
 *
 * Q, O: bf16 [B, Hq, Nq, d]; K, V: bf16 [B, Hkv, Nk, d]; LSE: fp32
 * [B, Hq, Nq].  Hq must be a multiple of Hkv: query head h reads key/value
 * head h / (Hq / Hkv) (Hkv = 1 is multi-query attention).  causal: query i
 * sees keys j <= i + (Nk - Nq), i.e. the last query is aligned with the last
 * key (for Nq == Nk this is the usual mask of fa_fwd).  A query row that sees
 * no key at all (causal with Nq > Nk) gets O = 0 and LSE = -inf.  B, Hq or
 * Nq equal to 0 is an empty problem (FA_OK, nothing launched); Nk = 0 with
 * queries present is FA_ERR_INVALID_ARG.  Otherwise as fa_fwd (fa_fwd is the
 * case Hq == Hkv, Nq == Nk).  One kernel launch on `stream`.
 */
int fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int Hq, int Hkv, int Nq,
              int Nk, int d, float scale, int causal, void* stream);

/* Workspace of fa_bwd_qk: as fa_bwd_workspace_size for the query side [B, Hq, Nq, d]. */
size_t fa_bwd_qk_workspace_size(int B, int Hq, int Nq, int d);

/*
 * Backward of fa_fwd_qk.  Q, O, dO: bf16 [B, Hq, Nq, d]; K, V: bf16
 * [B, Hkv, Nk, d]; LSE: fp32 [B, Hq, Nq] from fa_fwd_qk (read).  dQ: bf16
 * [B, Hq, Nq, d]; dK, dV: bf16 [B, Hkv, Nk, d], each the sum over the
 * Hq / Hkv query heads that read that key/value head (written).  workspace:
 * at least fa_bwd_qk_workspace_size(B, Hq, Nq, d) bytes.  Rows that see no key
 * contribute nothing and get dQ = 0.  Otherwise as fa_bwd (fa_bwd is the case
 * Hq == Hkv, Nq == Nk).
 */
int fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
              void* dK, void* dV, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Nq, int Nk,
              int d, float scale, int causal, void* stream);

/*
 * Forward over one block of keys, folded into running fp32 results, for
 * callers that attend one block of query rows to several key blocks in turn
 * (ring / context parallelism).  Q bf16 [B, Hq, Nq, d]; K, V bf16
 * [B, Hkv, Nk, d] (masked as fa_fwd_qk masks them).  O_acc fp32
 * [B, Hq, Nq, d] and LSE_acc fp32 [B, Hq, Nq] hold the result over the key
 * blocks folded so far; with this block's O_b, LSE_b the kernel writes
 * L = ln(exp(LSE_acc) + exp(LSE_b)), O_acc = exp(LSE_acc - L) O_acc +
 * exp(LSE_b - L) O_b, which is exact attention over the union of the blocks
 * (the per-row log-sum-exp that the online softmax uses across key tiles,
 * one level up).  first = 1 initialises the accumulators from this block
 * (their old contents are not read).  A side whose LSE is -inf weighs
 * nothing; rows that see no key in any block end with O_acc = 0, LSE_acc =
 * -inf.  No bf16 rounding happens between blocks.  One launch; checks and
 * status codes as fa_fwd_qk (first must be 0 or 1, every pointer 16-byte
 * aligned, the accumulators may not overlap the inputs).
 */
int fa_fwd_accumulate(const void* Q, const void* K, const void* V, float* O_acc, float* LSE_acc, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int causal, int first, void* stream);

/*
 * The backward in three steps, for callers that sum the gradients of one
 * block of query rows over several blocks of keys (ring / context
 * parallelism, where the key blocks arrive one at a time): the result over
 * the union of key blocks equals fa_bwd_qk over the whole key set, with no
 * rounding to bf16 between blocks.  The rows' O and LSE must be the final ones
 * over the whole key set (P is recomputed from LSE, and D from O and dO).
 *
 * fa_bwd_prepare: O, dO bf16 [B, Hq, Nq, d], LSE fp32 [B, Hq, Nq] (read).
 *   Writes D = rowsum(dO * O) and LSE * log2(e) into the workspace (at least
 *   fa_bwd_qk_workspace_size(B, Hq, Nq, d) bytes) and zeroes its fp32 dQ
 *   accumulator.  One launch.
 * fa_bwd_accumulate: Q, dO bf16 [B, Hq, Nq, d]; K, V bf16 [B, Hkv, Nk, d]
 *   (one key block, masked as fa_bwd_qk masks it: causal aligns the last
 *   query with the last key of THIS block).  Adds this block's dQ into the
 *   workspace accumulator; dK_acc, dV_acc fp32 [B, Hkv, Nk, d] receive the
 *   block's dK (scaled) and dV: stored when first = 1, added when first = 0.
 *   One launch; the workspace must come from fa_bwd_prepare of the same query
 *   block and must not be shared by calls that may overlap on the GPU.
 * fa_bwd_finish: dQ bf16 [B, Hq, Nq, d] = scale * the accumulated dQ.  One
 *   launch.
 * Same checks and status codes as fa_bwd_qk (first must be 0 or 1); every
 * pointer 16-byte aligned; outputs may not overlap inputs.
 */
int fa_bwd_prepare(const void* O, const void* dO, const float* LSE, void* workspace, size_t workspace_bytes, int B,
                   int Hq, int Nq, int d, void* stream);
int fa_bwd_accumulate(const void* Q, const void* K, const void* V, const void* dO, void* workspace,
                      size_t workspace_bytes, float* dK_acc, float* dV_acc, int B, int Hq, int Hkv, int Nq, int Nk,
                      int d, float scale, int causal, int first, void* stream);
int fa_bwd_finish(void* workspace, size_t workspace_bytes, void* dQ, int B, int Hq, int Nq, int d, float scale,
                  void* stream);

/*
 * Pieces of ring (context-parallel) attention, where each GPU holds one
 * chunk of the sequence and the key/value chunks travel around the ring of
 * GPUs (the pages name multi-card use for long contexts -- "NVIDIA Blackwell:
 * FlashAttention-4 Overcomes Memory Bottlenecks", body).  Exact attention
 * over the union of disjoint key sets follows from each set's O and LSE:
 * with L = ln(exp(LSE_a) + exp(LSE_b)), O = exp(LSE_a - L) O_a +
 * exp(LSE_b - L) O_b.
 *
 * fa_lse_merge folds one partial result (O_part bf16 [rows, d], LSE_part
 * fp32 [rows], as written by fa_fwd / fa_fwd_qk for the same query rows over
 * one key set) into an fp32 accumulator O_acc [rows, d] / LSE_acc [rows].
 * first = 1 initialises the accumulator from the partial (its old contents do
 * not matter).  A row whose LSE is -inf on one side takes the other side; -inf
 * on both gives O = 0, LSE = -inf.  d in {64, 128}.  O_part and O_acc 16-byte
 * aligned, the LSE arrays 4-byte aligned; the accumulator must not overlap the
 * partial.  One kernel launch on `stream`.
 */
int fa_lse_merge(const void* O_part, const float* LSE_part, float* O_acc, float* LSE_acc, int64_t rows, int d,
                 int first, void* stream);

/* acc (fp32, n) = (first ? 0 : acc) + x (bf16, n); n a multiple of 8, both 16-byte aligned. */
int fa_accumulate_bf16(float* acc, const void* x, int64_t n, int first, void* stream);

/*
 * acc (fp32, n) += x (fp32, n), elementwise: adds one step's gradient block to
 * an accumulator (ring backward).  n a multiple of 8, both 16-byte aligned,
 * not overlapping.  One launch on `stream`.
 */
int fa_accumulate_f32(float* acc, const float* x, int64_t n, void* stream);

/* y (bf16, n) = x (fp32, n) rounded to nearest even; n a multiple of 8, both 16-byte aligned. */
int fa_convert_f32_bf16(const float* x, void* y, int64_t n, void* stream);

/* Static human-readable text for a status code. */
const char* fa_strerror(int status);

/*
 * Synchronises `stream`, then reports device-side failures since the last
 * call on the current device: FA_ERR_TIMEOUT if a kernel's bounded wait
 * expired (the detail code, kernel and wait site, is returned through
 * *detail when detail is not NULL), FA_ERR_CUDA if the synchronisation
 * itself failed, FA_OK otherwise.  Clears the recorded failure.
 */
int fa_last_device_status(void* stream, int* detail);

/*
 * Tuning of the forward softmax (process-wide; for A/B comparisons).
 * tau: rescale threshold in log2 units (0 <= tau <= 16; 0 = rescale whenever
 * the running maximum grows; default 8).  poly: how many of every 16 element
 * pairs of an interior tile take the FMA-pipe cubic exp2 instead of the SFU:
 * 0 (all on the SFU), 1, 2 or 4 (a sixteenth, an eighth, a quarter); -1
 * restores the library's default for each head dimension.  Returns
 * FA_ERR_INVALID_ARG for values out of range.
 *
 * This and the two variant setters below change process-wide settings.  They
 * are safe to call from any thread, but a call of fa_fwd* / fa_bwd* running
 * at the same time on another thread may see the old or the new setting: set
 * them between calls.
 */
int fa_set_softmax_options(float tau, int poly);

/*
 * Forward kernel selection (process-wide; for A/B comparisons).  0 (default):
 * the single-CTA kernel.  1: at d = 128 the forward runs on cluster pairs of
 * SMs, every MMA a 2-SM (cta_group::2) UMMA of M = 256 with K and V split
 * between the pair (same results, currently slower).  d = 64 always uses the
 * single-CTA kernel.
 * Returns FA_ERR_INVALID_ARG for other values.
 */
int fa_set_forward_variant(int cluster_pair);

/*
 * Backward kernel selection (process-wide; for A/B comparisons).  0: the
 * single-CTA kernel.  1: at d = 128, for one query head per key/value head and
 * Nq == Nk, the backward runs on cluster pairs of SMs that own two adjacent
 * key tiles ("C. Le Duo de Cuisiniers (2-CTA)", FlashAttention-4 pages): every
 * MMA is a 2-SM (cta_group::2) UMMA, the query-tile operands are split between
 * the pair, and dQ of a query tile is summed over both key tiles on chip
 * (each CTA hands the other half of its dS).  Same results, currently slower
 * (0 is the default); other shapes always use the single-CTA kernel.
 * Returns FA_ERR_INVALID_ARG for other values.
 */
int fa_set_backward_variant(int cluster_pair);

/*
 * Elementwise y = 2^x on the device for testing the exponential the kernels
 * use: mode 0 = the cubic-polynomial software exp2, mode 1 = the SFU
 * (ex2.approx), mode 2 = the cubic with packed fp32x2 arithmetic on element
 * pairs (must equal mode 0 bit for bit).  x, y: fp32 device arrays of n
 * elements, 16-byte aligned.
 */
int fa_exp2_eval(const float* x, float* y, int64_t n, int mode, void* stream);

/*
 * Profiling hook (used by the benchmark to time one kernel inside a call):
 * when start_event and stop_event are cudaEvent_t handles, the NEXT fa_fwd*
 * (which = 0) or fa_bwd* (which = 1) call made on the SAME host thread
 * records start_event on its stream immediately before its main attention
 * kernel and stop_event immediately after it, then forgets both.  Requests
 * are per thread, so calls on other threads neither see nor consume them.
 * NULL, NULL clears a pending request.  Returns FA_ERR_INVALID_ARG for
 * another `which` or a half-NULL pair.
 */
int fa_profile_next(int which, void* start_event, void* stop_event);

/*
 * SM clock probe (used by the benchmark to state the clock the kernels ran
 * at): launches one single-thread kernel on `stream` that counts SM cycles
 * (clock64) while the global nanosecond timer advances by about 20 us, and
 * writes out[0] = cycles, out[1] = nanoseconds; the effective SM clock is
 * 1000 * out[0] / out[1] MHz at the moment the probe runs (for example right
 * after an attention kernel, before the power manager reacts).  `out` is a
 * device array of two uint64, 8-byte aligned.  Returns the launch status.
 */
int fa_sm_clock_probe(uint64_t* out, void* stream);

/*
 * Failure-path self test: launches one small kernel on `stream` whose only
 * pipeline wait is on a barrier that nothing ever arrives at.  The bounded
 * wait used by every kernel of the library gives up after its limit (2 s),
 * records its site in the device status word and the kernel returns; no
 * fault, trap or hang is involved.  A following fa_last_device_status(stream)
 * must then report FA_ERR_TIMEOUT with detail 0xF01.  Returns the launch
 * status.
 */
int fa_selftest_wait_timeout(void* stream);

/* Size of the fixed device scratch array behind fa_bwd_noalloc (64 MiB). */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * fa_bwd_noalloc -- the backward pass for callers that cannot allocate
 * device memory.  The paper has no counterpart; this entry point exists for
 * integration only.  Some callers of this library cannot call cudaMalloc:
 * for example a serving process whose memory manager has already reserved
 * the whole device, or latency-critical code that must not pay for
 * cudaMalloc's implicit device-wide synchronisation.  fa_bwd needs a caller
 * workspace; this variant instead uses a scratch array of
 * FA_BWD_NOALLOC_SCRATCH_BYTES that is a file-scope __device__ variable of
 * the library, so every GPU that loads the library holds it until the
 * process exits.  The caller still passes all inputs and outputs, with the
 * same meaning, layout and checks as fa_bwd; nothing is allocated by the
 * call (no cudaMalloc, cudaFree or allocating library routine).
 *
 * Limit: the problem must satisfy fa_bwd_workspace_size(B, H, N, d) <=
 * FA_BWD_NOALLOC_SCRATCH_BYTES, i.e. B*H*ceil(N/128)*128 <= 129,024 rows at
 * d = 128 (e.g. B*H = 16 heads of N = 8064) and <= 254,080 rows at d = 64;
 * larger problems return FA_ERR_UNSUPPORTED before anything is launched.  The first call on a device looks up the scratch array's
 * device address (cudaGetSymbolAddress, once per device, with that device
 * current); make that first call before any stream capture.  Every call
 * shares the one array and leaves its contents behind; each call clears
 * what must start at zero itself.  Calls whose GPU work overlaps (different
 * streams, or different host threads, on the same device) race on the
 * scratch and give wrong results: serialise them.
 */
int fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                   void* dQ, void* dK, void* dV, int B, int H, int N, int d, float scale, int causal,
                   void* stream);

/* Library version, 100 * major + minor. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
