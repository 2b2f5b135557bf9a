/*
 * fa.h -- C ABI of the B200 (sm_100a) exact IO-aware attention library.
 *
 * What the library computes is exact attention, O = softmax(scale * Q K^T) V,
 * tiled so that the N x N scores S and probabilities P live only in on-chip
 * memory (TMEM / shared memory) and are never written to HBM; the forward saves
 * one per-row statistic and the backward recomputes P tile by tile from it.
 * Sources: explainers.rudrite.com "flash-attention-anatomy" (Q&As "Why is
 * attention memory-bound, and how does FlashAttention fix it?", "What is online
 * softmax and how does tiling keep it exact?", "How does FlashAttention save
 * memory in the backward pass?", "What changed between FlashAttention 1, 2, and
 * 3?"); chipfoundryservices.com glossary "flash attention" ("Tiling plus an
 * online softmax removes the round trip"); kipu-akw.pages.dev "flash-attention /
 * where-it-matters" (section "The Real Complexity").
 *
 * Conventions shared by every entry point:
 *   - Layout: contiguous [B, H, N, d] row-major, d innermost, for every
 *     [.., N, d] tensor; LSE and other per-row values are contiguous [B, H, N].
 *   - Device pointers.  The caller owns every buffer (including the backward
 *     workspace); the library allocates no device or pinned memory, keeps no
 *     pointer after a call returns, and never synchronises the stream.
 *   - Tensor pointers (q, k, v, o, dO, dq, dk, dv, workspace) must be 16-byte
 *     aligned; lse must be 4-byte aligned.
 *   - d (head dimension) must be 64 or 128.  N >= 1 is arbitrary: ragged tails
 *     are masked.  B, H, N == 0 is a valid empty call that launches nothing.
 *   - causal != 0 selects top-left aligned causal masking (key j is visible to
 *     query i iff j <= i; Nq == Nk == N).  Fully masked tiles are skipped.
 *   - scale is the softmax scale (the configurations use 1/sqrt(d)).  It must
 *     be finite and >= 0; scale = 0 is valid and makes every visible key
 *     equally weighted (O is the mean of the visible V rows, LSE = ln of
 *     their count, dQ = dK = 0).  A negative or non-finite scale returns
 *     FA_ERR_INVALID_ARG.
 *   - stream is a cudaStream_t passed as an opaque pointer (NULL = legacy
 *     default stream).
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns an error code and launches nothing.  A launch failure
 *     returns FA_ERR_LAUNCH.  Asynchronous device faults surface at the
 *     caller's next synchronisation.  Every device-side wait is bounded; one
 *     that runs out records a status readable with fa_device_status().
 *   - Thread safety: calls are re-entrant; the first call on a device also
 *     configures the kernels' shared-memory limits for that device.
 *   - CUDA graphs: the attention calls (fa_fwd*, fa_bwd*, fa_fwd_decode,
 *     fa_fwd_standard) only enqueue kernel launches on the stream, so a
 *     caller may capture them into a graph and replay it.  Make the first
 *     call on each device outside any capture (it looks up device attributes
 *     and symbol addresses once).  fa_bwd_events also records the caller's
 *     events, which time nothing inside a capture; fa_device_status
 *     synchronises and cannot be captured.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null pointer, bad size or dimension, bad scale */
  FA_ERR_UNSUPPORTED = 2,     /* head dimension other than 64 / 128 */
  FA_ERR_ALIGNMENT = 3,       /* pointer not 16-byte (4-byte for lse) aligned */
  FA_ERR_ARCH = 4,            /* current device is not sm_100 (B200 class) */
  FA_ERR_LAUNCH = 5,          /* CUDA runtime rejected a launch or attribute */
  FA_ERR_DEVICE_TIMEOUT = 6,  /* a bounded device wait ran out (fa_device_status) */
  FA_ERR_WORKSPACE = 7,       /* backward workspace missing or too small */
  FA_ERR_SCRATCH_LIMIT = 8    /* shape needs more than fa_bwd_noalloc's fixed scratch */
} fa_status;

/*
 * Forward pass, bf16.
 * Computes O = softmax(scale * Q K^T) V per (batch, head) with a running row
 * maximum m and denominator l carried across key tiles and the partial output
 * rescaled by exp(m_old - m_new) when m grows ("What is online softmax and how
 * does tiling keep it exact?"); writes only O and LSE = m + ln l, never S or P
 * ("How does FlashAttention save memory in the backward pass?": the per-row
 * softmax statistics are the only residual).
 *   q, k, v : in,  bf16 [B,H,N,d]
 *   o       : out, bf16 [B,H,N,d]
 *   lse     : out, fp32 [B,H,N], natural-log log-sum-exp of each score row
 */
FA_API fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for this shape (0 when empty).
 * The workspace holds D = rowsum(dO o O) and the log2-domain LSE, both fp32
 * per row padded to a multiple of 128 rows, and the fp32 dQ accumulator.
 * Returns (size_t)-1 when the arguments are invalid.
 */
FA_API size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass, bf16, for a loss L with dL/dO = dO.
 * Recomputes S and P = exp(S - LSE) tile by tile from Q, K and the saved LSE
 * instead of reading a stored P ("How does FlashAttention save memory in the
 * backward pass?"; "The Real Complexity", recomputation on the backward pass),
 * then forms D = rowsum(dO o O), dV = P^T dO, dP = dO V^T, dS = P o (dP - D),
 * dQ = scale dS K, dK = scale dS^T Q (chain rule through S = scale Q K^T).
 * dQ is accumulated across key tiles with fp32 atomics, so its low bits may
 * differ from run to run.
 *   q, k, v, o, dO : in,  bf16 [B,H,N,d]  (o: the forward's output)
 *   lse            : in,  fp32 [B,H,N]    (the forward's LSE)
 *   dq, dk, dv     : out, bf16 [B,H,N,d]
 *   workspace      : scratch device memory of >= workspace_bytes bytes, at
 *                    least fa_bwd_workspace_size(B,H,N,d); contents on entry
 *                    are ignored and on exit are unspecified.  Must not be
 *                    used by another call that overlaps this one on the GPU.
 */
FA_API fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                 void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd with per-launch timing: the same computation, arguments and errors
 * as fa_bwd, and additionally records four CUDA events (cudaEvent_t values
 * passed as opaque pointers, created by the caller) on `stream`:
 *   events[0] before the preprocess launch (D = rowsum(dO o O)),
 *   events[1] before the recompute kernel (S, P, dV, dP, dS, dK, dQ),
 *   events[2] after it, before the dQ conversion to bf16,
 *   events[3] after the last launch.
 * The elapsed time between events[1] and events[2] is the main kernel's own
 * duration on the launching stream.  Any NULL event returns
 * FA_ERR_INVALID_ARG before anything is launched.
 */
FA_API fa_status fa_bwd_events(const void* q, const void* k, const void* v, const void* o, const void* dO,
                               const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                               float scale, int causal, void* workspace, size_t workspace_bytes,
                               void* const* events, void* stream);

/*
 * Backward pass with a deterministic dQ: same arguments, outputs and workspace
 * as fa_bwd, but dQ is produced by a separate query-tile-parallel pass that
 * recomputes S, P and dP per query tile and accumulates dQ_i += dS K_j in
 * on-chip memory, writing each row once (no atomics).  Repeated calls on the
 * same inputs return bit-identical dQ, dK and dV.  Costs two more GEMMs per
 * tile pair (the recomputed S and dP) than fa_bwd.
 */
FA_API fa_status fa_bwd_deterministic(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                      const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                                      float scale, int causal, void* workspace, size_t workspace_bytes,
                                      void* stream);

/*
 * Launch plan of fa_fwd and fa_fwd_fp8 for a shape, computed on the host as
 * the forward computes it (no launch; uses the current device's SM count, or
 * 148 when no device is visible).  A work item is one 128-row Q tile or a
 * pair of them of one (batch, head):
 *   *ctas       : CTAs launched (d = 64 non-causal runs at most one
 *                 persistent CTA per SM over the items)
 *   *items      : work items
 *   *pair_items : items that hold a pair of Q tiles; on non-causal grids the
 *                 pairs of a last round that would fill at most half of the
 *                 SMs are split into single-tile items dispatched last.
 * scale is not an argument; the other arguments are checked as in fa_fwd.
 */
FA_API fa_status fa_fwd_plan(int B, int H, int N, int d, int causal, int* ctas, int* items, int* pair_items);

/*
 * Forward pass with float8 e4m3 inputs and per-tensor scales ("What changed
 * between FlashAttention 1, 2, and 3?": low-precision FP8 forward).
 * The real inputs are q8 * q_descale, k8 * k_descale, v8 * v_descale.  The
 * score and value descales are folded into the exponent argument and the
 * final normalisation; P is rounded to e4m3 for the P V product while the
 * denominator l is summed in fp32.
 *   q8, k8, v8 : in,  e4m3 (fn) bytes [B,H,N,d]
 *   o          : out, bf16 [B,H,N,d]
 *   lse        : out, fp32 [B,H,N]
 * d must be 128 (a head row is one 128-byte swizzle span); causal is supported.
 */
FA_API fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale, float k_descale,
                     float v_descale, void* o, float* lse, int B, int H, int N, int d, float scale, int causal,
                     void* stream);

/*
 * Backward pass of fa_fwd_fp8: gradients with respect to the real inputs
 * q8 * q_descale, k8 * k_descale, v8 * v_descale of the e4m3 forward
 * ("What changed between FlashAttention 1, 2, and 3?" names low-precision
 * FP8 as the forward's speed lever; the backward is the chain rule of the same
 * attention, as in fa_bwd).
 * Every e4m3 value is exactly a bf16 value, so the e4m3 Q, K and V are first
 * widened to bf16 in the workspace (no rounding) and the bf16 backward
 * kernels run on them; the descales are folded into the score factor
 * (scale * q_descale * k_descale), into dP (v_descale), dK (scale * q_descale)
 * and dQ (scale * k_descale).  The probabilities P and the gradient dS stay
 * bf16: normalised P is about 1/N (below e4m3's smallest subnormal, 2^-9, at
 * N >= 1024 with diffuse attention) and dS has a data-dependent range, so
 * neither fits a per-tensor e4m3 scale.
 *   q8, k8, v8 : in,  e4m3 (fn) bytes [B,H,N,d] (the forward's inputs)
 *   o          : in,  bf16 [B,H,N,d] (fa_fwd_fp8's output)
 *   dO         : in,  bf16 [B,H,N,d]
 *   lse        : in,  fp32 [B,H,N] (fa_fwd_fp8's LSE)
 *   dq, dk, dv : out, bf16 [B,H,N,d], in the real (descaled) units
 *   workspace  : >= fa_bwd_fp8_workspace_size(B,H,N,d) bytes (fa_bwd's
 *                workspace plus the three widened tensors, 6 N d bytes per head)
 * d must be 128 (as fa_fwd_fp8); causal is supported; descales must be
 * finite and > 0.  dQ is reduced with fp32 atomics as in fa_bwd.
 */
FA_API fa_status fa_bwd_fp8(const void* q8, const void* k8, const void* v8, float q_descale, float k_descale,
                            float v_descale, const void* o, const void* dO, const float* lse, void* dq, void* dk,
                            void* dv, int B, int H, int N, int d, float scale, int causal, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Bytes of workspace fa_bwd_fp8 needs ((size_t)-1 for invalid arguments or d != 128). */
FA_API size_t fa_bwd_fp8_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass for callers that cannot allocate device memory.  The pages
 * have no counterpart: this is a packaging variant of fa_bwd, not a step of
 * the method.  Some callers cannot call cudaMalloc where they run the
 * backward -- a plugin inside a framework that owns every device allocation
 * and gives the plugin no allocator, or a serving loop that reserves its
 * memory at start-up and must not allocate (or risk a device-wide
 * synchronisation) afterwards.  This entry point takes the same arguments as
 * fa_bwd minus the workspace, and allocates nothing: its scratch is a fixed
 * array of fa_bwd_noalloc_max_bytes() bytes (64 MiB) inside the library,
 * which every GPU that loads the library holds until the process exits.
 *   - Shapes whose fa_bwd_workspace_size() exceeds that limit are rejected
 *     with FA_ERR_SCRATCH_LIMIT before anything is launched.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; the
 *     part that must start at zero is cleared by each call itself.  Calls
 *     whose GPU work overlaps (other streams, unordered host threads) race
 *     on it and must be serialised by the caller.
 */
FA_API fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                                float scale, int causal, void* stream);

/* Size in bytes of fa_bwd_noalloc's fixed scratch array. */
FA_API size_t fa_bwd_noalloc_max_bytes(void);

/*
 * Decode against a KV cache: Nq (1..16) new queries per (batch, head) attend
 * over Nk cached keys (chipfoundryservices glossary "flash attention", closing
 * section: the method serves inference against a KV cache).  The key range is split
 * across CTAs; each split keeps its own running max and sum, and the splits
 * are combined by their log-sum-exp (O = sum_s exp(LSE_s - LSE) O_s).  HBM-
 * bound: K and V are read once.
 *   q      : in,  bf16 [B,H,Nq,d]
 *   k, v   : in,  bf16 [B,H,Nk,d]
 *   o      : out, bf16 [B,H,Nq,d]
 *   lse    : out, fp32 [B,H,Nq]
 *   causal : query i of the Nq sees keys j <= Nk - Nq + i (the queries are the
 *            last Nq positions of the sequence); needs Nk >= Nq.
 *   workspace : >= fa_fwd_decode_workspace_size(B,H,Nq,Nk,d) bytes of device
 *            scratch for the per-split partial results (may be NULL when that
 *            size is 0 or the plan uses a single split).
 * Errors: FA_ERR_UNSUPPORTED for Nq > 16 or d not in {64,128};
 * FA_ERR_INVALID_ARG for Nk == 0 (with queries) or causal with Nk < Nq.
 */
FA_API fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                               int Nq, int Nk, int d, float scale, int causal, void* workspace,
                               size_t workspace_bytes, void* stream);

/* Bytes of workspace fa_fwd_decode needs ((size_t)-1 for invalid arguments). */
FA_API size_t fa_fwd_decode_workspace_size(int B, int H, int Nq, int Nk, int d);

/*
 * Standard (materialising) attention, the baseline the method is measured
 * against (explainers.rudrite.com "flash-attention-anatomy", Q&A "Why is
 * attention memory-bound, and how does FlashAttention fix it?": S is written
 * to HBM, read back for the softmax, P written, and read again for P V).
 * Same arguments and results as fa_fwd (O bf16, LSE fp32 natural log, causal
 * top-left aligned), computed in three passes through the workspace:
 *   S = scale Q K^T   fp32 [B,H,N,Np]   (Np = N rounded up to 128)
 *   P = softmax(S)    bf16 [B,H,N,Np]   (normalised; causal mask applied here)
 *   O = P V
 * workspace: >= fa_fwd_standard_workspace_size(B,H,N,d) bytes of device
 * memory, 256-byte aligned; about 6 N^2 bytes per head.
 */
FA_API fa_status fa_fwd_standard(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                                 int N, int d, float scale, int causal, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Bytes of workspace fa_fwd_standard needs ((size_t)-1 for invalid arguments). */
FA_API size_t fa_fwd_standard_workspace_size(int B, int H, int N, int d);

/* Human-readable text for a status code (static storage, never NULL). */
FA_API const char* fa_strerror(fa_status status);

/*
 * Reads and clears the library's device status word on the current device.
 * Synchronises `stream` first.  Returns FA_OK, or FA_ERR_DEVICE_TIMEOUT if a
 * bounded wait inside a kernel ran out since the last call (the kernel then
 * abandoned its tile and returned; its outputs are undefined).  *where, if
 * not NULL, receives a code naming the wait that gave up.
 */
FA_API fa_status fa_device_status(void* stream, uint32_t* where);

/*
 * fa_device_status(stream, NULL): the device status check without the code
 * of the wait site.
 */
FA_API fa_status fa_get_device_status(void* stream);

/*
 * Self-test of the bounded-wait machinery: launches one block that waits on a
 * barrier nobody arrives at, with the given limit in microseconds (1..10^6),
 * so the wait runs out and the status word is set.  Used by the tests to
 * check that a stuck wait ends with a status, not a hang.
 */
FA_API fa_status fa_watchdog_selftest(uint32_t limit_us, void* stream);

/* Library version as major*10000 + minor*100 + patch. */
FA_API int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
