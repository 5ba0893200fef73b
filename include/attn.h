/* attn.h -- C ABI of the B200 exact-attention library (libattn_b200.so).
 *
 * The operation is exact scaled-dot-product attention,
 *     O = softmax(scale * Q K^T) V,
 * as defined on page "attention 的显存线性化" §一 (softmax(Q K^T / sqrt(d_k)) V)
 * and page "注意力计算的计算与显存瓶颈" §1.1.1 (S = Q K^T / sqrt(d), P = softmax(S),
 * O = P V), computed tile by tile with an online softmax so that the n x n
 * matrices S and P never reach device memory (page "attention 的显存线性化" §三;
 * page "attn-efficient", online-softmax section).  The backward recomputes the
 * needed S/P tiles from the saved log-sum-exp instead of storing them (page
 * "attention 的显存线性化" §五; page "attn-efficient", recompute paragraph).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers: all tensor pointers are DEVICE pointers on the current CUDA device,
 *   owned by the caller, contiguous row-major, 16-byte aligned.  The library
 *   keeps no pointer after a call returns.
 * Layouts (bf16 = IEEE bfloat16, 2 bytes; fp32 = 4 bytes):
 *   q, o, dO, dq : bf16 [B][Hq][N][d]
 *   k, v, dk, dv : bf16 [B][Hkv][N][d]
 *   lse          : fp32 [B][Hq][N], natural log of sum_j exp(scale * q_i . k_j)
 *                  over the keys row i may see.
 * Heads: grouped-query attention maps q-head h to kv-head h / (Hq / Hkv)
 *   (contiguous groups; page "attn-efficient", GQA / MQA row of the family table).
 *   Hkv == Hq is ordinary multi-head attention, Hkv == 1 is multi-query attention.
 * causal: 0 = every query sees every key; 1 = query i sees keys j <= i
 *   (equal query and key lengths).
 * scale: finite and >= 0; the usual value is 1/sqrt(d).
 * d: 64 or 128.  N: any value >= 1 (ragged tails are masked on device).
 * Streams: work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *   stream) and the call returns without waiting.  Results are stream-ordered.
 * Errors: arguments are validated on the host before any launch; a rejected
 *   call launches nothing and returns a negative attn_status_t.  Device-side
 *   waits are bounded: if one expires the kernel records an error word and
 *   exits; attn_get_device_status() reports it.  No entry point aborts, traps
 *   or throws.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,   /* null pointer, bad shape, Hq % Hkv != 0, bad scale */
  ATTN_ERR_UNSUPPORTED = -2,   /* d not in {64, 128}, or no sm_100 device */
  ATTN_ERR_ALIGNMENT = -3,     /* a pointer is not 16-byte aligned */
  ATTN_ERR_LAUNCH = -4,        /* the CUDA runtime refused a launch or an attribute */
  ATTN_ERR_DEVICE_TIMEOUT = -5,/* a bounded device wait expired (see attn_get_device_status) */
  ATTN_ERR_WORKSPACE = -6,     /* backward workspace too small (or beyond the no-alloc scratch) */
  ATTN_ERR_ALLOC = -7,         /* the library's own stream-ordered allocation failed */
  ATTN_ERR_DEVICE_BOUNDS = -8, /* checking build only: a kernel computed an index outside its tensor */
  ATTN_ERR_SCHED_CONFLICT = -9 /* more than 128 forward/decode launches in flight: one stopped early */
} attn_status_t;

/* Forward: O and LSE for every (b, h, i).
 * Reads q, k, v; writes o and lse.  Returns ATTN_OK or a negative status.
 * Enqueues two kernels on `stream`: a one-thread kernel that zeroes this call's
 * work counter, then the forward, whose persistent CTAs claim work units from
 * that counter.  Each call takes the next of 128 counters (rotating, shared with
 * attn_fwd_window, attn_fwd_fp8 and attn_decode), so up to 128 such calls may be in
 * flight at once, on any streams.  Beyond that, a call whose counter is taken over
 * by a later one stops claiming work and ATTN_ERR_SCHED_CONFLICT is reported through
 * attn_get_device_status(); the outputs of both calls are then incomplete (a stale
 * claim may also use up one of the later call's work units). */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
             void* stream);

/* FP8 forward: as attn_fwd with Q, K and V in e4m3 (OCP FP8: 1 sign, 4 exponent
 * bits with bias 7, 3 mantissa bits; one byte each, same [B][H][N][d] layouts) and
 * per-tensor descales: the values attended to are q * q_descale, k * k_descale and
 * v * v_descale.  Both products run on the tensor cores with 8-bit operands
 * (tcgen05 kind::f8f6f4): S from the e4m3 Q and K, and O from P rounded to e4m3
 * (round to nearest even; P <= 256 by the lazy rescale) times the e4m3 V.  The row
 * sums and the LSE use the unrounded P, as in attn_fwd.  O is bf16, lse fp32
 * (page "attention 的显存线性化" §五 names FP8 support for the later versions; the
 * pages give no recipe, so the per-tensor descales are this library's reading).
 * d is 64 or 128 (a 64-byte e4m3 row is zero-padded to the 128-byte swizzle row on
 * chip; ATTN_ERR_UNSUPPORTED otherwise); descales finite and > 0. */
int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int N, int d, float scale,
                 float q_descale, float k_descale, float v_descale, int causal, void* stream);

/* Local (sliding-window) forward: as attn_fwd, but query i sees only keys j with
 *     i - window_left <= j <= i + window_right
 * (page "attn-efficient", sliding-window row of the efficient-attention family
 * table: each position attends to the w positions nearest it, O(n*w) work).  A
 * negative side means no limit on that side, so (-1, 0) is causal attention,
 * (-1, -1) full attention, (w - 1, 0) a causal window of w keys and (w, w) a
 * symmetric one.  Key tiles outside every row's band are skipped, so the work
 * grows with N * (window_left + window_right + 1).  Same layouts, errors and
 * stream behaviour as attn_fwd. */
int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int Hq, int Hkv, int N, int d, float scale,
                    int window_left, int window_right, void* stream);

/* Bytes of device workspace attn_bwd needs for this shape (8 bytes per query row:
 * the row's log-sum-exp in log2 units and D_i = sum_k dO_ik O_ik, both fp32; rows
 * padded to a multiple of 128).  Contents need no initialisation.  Returns 0 for
 * arguments attn_bwd would reject. */
size_t attn_bwd_workspace_size(int B, int Hq, int Hkv, int N, int d, int causal);

/* Backward: gradients of sum(O * dO) with respect to q, k, v.
 * Reads q, k, v, o (the forward output), lse (the forward log-sum-exp) and dO;
 * writes dq, dk, dv.  For GQA, dk and dv sum over the q-heads of each group.
 * The reduction order is fixed, so two calls on the same inputs give the same
 * bits.
 * Workspace ownership: if `workspace` is non-NULL it must hold
 *   attn_bwd_workspace_size(...) bytes (else ATTN_ERR_WORKSPACE), 16-byte aligned
 *   (else ATTN_ERR_ALIGNMENT); it is overwritten and stays the caller's.  If it is
 *   NULL (`workspace_bytes` is then ignored), the library takes the workspace
 *   with cudaMallocAsync on `stream` and releases it with cudaFreeAsync on
 *   `stream` behind its kernels, so the call stays asynchronous; a failed
 *   allocation returns ATTN_ERR_ALLOC with nothing launched. */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* dO, void* dq, void* dk, void* dv,
             int B, int Hq, int Hkv, int N, int d, float scale, int causal,
             void* workspace, size_t workspace_bytes, void* stream);

/* Backward of attn_fwd_window: gradients of sum(O * dO) for the same band of
 * visible keys (window_left / window_right as in attn_fwd_window; o and lse must
 * come from attn_fwd_window with the same window).  Workspace and stream rules
 * are those of attn_bwd; attn_bwd_workspace_size does not depend on the mask. */
int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv,
                    int B, int Hq, int Hkv, int N, int d, float scale,
                    int window_left, int window_right,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Decoding: Nq new query rows against Nk keys (a KV cache), split over the keys
 * (page "attention 的显存线性化", reading list: FlashDecoding).  The keys of each
 * (batch, kv-head) are cut into splits processed in parallel; each split leaves a
 * partial output and log-sum-exp, and the partials are merged with the online-
 * softmax rescale (page "attn-efficient", online-softmax section):
 * O = sum_s exp(LSE_s - LSE) O_s.  The result is exact attention over all Nk keys.
 *   q, o : bf16 [B][Hq][Nq][d]     k, v : bf16 [B][Hkv][Nk][d]     lse : fp32 [B][Hq][Nq]
 *   causal: 1 = the queries are the last Nq positions of the sequence: query i
 *     sees keys j <= Nk - Nq + i (requires Nq <= Nk); 0 = every query sees every key.
 *   Hq / Hkv <= 128 (the group's query heads share one K/V stream).
 * Workspace (the split partials): attn_decode_workspace_size(...) bytes, queried
 * with the same device current (the split count depends on its SM count; 0 when
 * one split suffices).  NULL: the library allocates it on `stream` with
 * cudaMallocAsync / cudaFreeAsync.  Errors as attn_fwd, plus ATTN_ERR_WORKSPACE
 * (too small) and ATTN_ERR_ALLOC.  Enqueues a counter-reset kernel, the split
 * kernel and, with more than one split, the merge kernel. */
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);
int attn_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal,
                void* workspace, size_t workspace_bytes, void* stream);
/* Number of key splits attn_decode uses for this shape on the current device
 * (0 for arguments it would reject). */
int attn_decode_splits(int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal);

/* Merge of a partial attention result into a running one, for keys that arrive in
 * blocks -- e.g. sequence shards passed around a ring of GPUs (the online-softmax
 * rescale of page "attn-efficient" applied to whole blocks):
 *   m = max(lse_acc, lse_part), a = exp(lse_acc - m), b = exp(lse_part - m),
 *   o_acc = (a o_acc + b o_part) / (a + b),  lse_acc = m + ln(a + b).
 *   o_acc  : fp32 [rows][d], updated in place (its contents are ignored where lse_acc = -inf)
 *   lse_acc: fp32 [rows], updated in place; initialise to -inf for an empty accumulator
 *   o_part : bf16 [rows][d] and lse_part fp32 [rows] -- an attn_fwd / attn_decode result
 *   out    : NULL, or bf16 [rows][d] that receives the merged O rounded to bf16
 * d is 64 or 128.  One kernel on `stream`. */
int attn_merge(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
               long long rows, int d, void* out, void* stream);

/* Accumulation of a gradient contribution in fp32, for gradients summed over key or
 * query blocks -- e.g. the backward over a ring of GPUs, where each step's attn_bwd
 * returns one block pair's dQ, dK, dV (no counterpart on the pages; the plain sum of
 * the per-block gradients that the recompute backward of page "attention 的显存线性化"
 * §五 implies when the keys are split into blocks):
 *   acc[i] += part[i] for 0 <= i < n.
 *   acc : fp32 [n], updated in place;  part : bf16 [n].
 * n is a multiple of 8 (>= 8); both pointers 16-byte aligned.  One kernel on `stream`.
 * The sum is taken in fp32 in the order of the calls, so a fixed call order gives a
 * bitwise reproducible result. */
int attn_accumulate(float* acc, const void* part, long long n, void* stream);

/* Backward without a caller-provided workspace (no counterpart on the pages; an
 * interface convenience).  Same arguments, layouts and results as attn_bwd, minus
 * `workspace`/`workspace_bytes`: the scratch lives in a fixed 64 MiB device array
 * owned by this library (held on every GPU that loads the library, until exit).
 * For callers that cannot call cudaMalloc -- e.g. code running inside a host
 * framework whose memory pool owns all device memory, or a loop that must not
 * allocate after start-up -- this call allocates nothing and calls no allocating
 * routine.
 *   - Shapes whose workspace (attn_bwd_workspace_size) exceeds 64 MiB
 *     (67108864 bytes) are rejected with ATTN_ERR_WORKSPACE before any launch.
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.  If
 *     that lookup fails the call returns ATTN_ERR_LAUNCH and the next call
 *     tries the lookup again.
 *   - All calls share the one array and leave their contents in it; everything
 *     that must start at zero is cleared by the call itself.  Calls that overlap
 *     on the GPU (different streams, or different host threads) race on the
 *     array: serialise them. */
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                     const void* dO, void* dq, void* dk, void* dv,
                     int B, int Hq, int Hkv, int N, int d, float scale, int causal,
                     void* stream);

/* Synchronises `stream`, then returns ATTN_OK if no kernel of this library
 * recorded a device-side error since the last call, else ATTN_ERR_DEVICE_TIMEOUT
 * (a bounded wait expired), ATTN_ERR_DEVICE_BOUNDS (checking build: an index
 * check failed) or ATTN_ERR_SCHED_CONFLICT (see attn_fwd); the error word is cleared.  While the word is set, later launches
 * exit early. */
int attn_get_device_status(void* stream);

/* Static, human-readable text for a status code. */
const char* attn_status_string(int status);

/* Checking build (no counterpart on the pages).  The library also comes as
 * libattn_b200_checks.so, compiled with ATTN_CHECKS: its kernels test every tile
 * coordinate, head index and global row they compute against the tensor it
 * addresses; an index out of range records ATTN_ERR_DEVICE_BOUNDS in the error word
 * and the access is skipped or kept inside the tensor -- no trap, no assert.  It
 * stands in for a memory checker where none can run.
 * attn_checks_enabled returns 1 in that build, 0 in the normal one.
 * attn_selftest_bounds launches one CTA that hands the check an index outside its
 * range (nothing is accessed with it): in the checking build the following
 * attn_get_device_status() returns ATTN_ERR_DEVICE_BOUNDS, in the normal build
 * ATTN_OK.  Returns ATTN_ERR_LAUNCH if the launch is refused, else ATTN_OK. */
int attn_checks_enabled(void);
int attn_selftest_bounds(void* stream);

/* Diagnostic (no counterpart on the pages): exercises the device-side failure
 * path that every kernel of this library uses.  Launches one CTA on `stream`
 * that waits on an mbarrier nothing will ever arrive on, through the same bounded
 * wait as the kernels but with a limit of `limit_ns` nanoseconds (1 ns .. 1 s).
 * The wait gives up, records the timeout in the error word and the CTA returns:
 * nothing hangs, traps or faults.  A following attn_get_device_status() returns
 * ATTN_ERR_DEVICE_TIMEOUT and clears the word.  Returns ATTN_ERR_INVALID_ARG for
 * a limit out of range, ATTN_ERR_LAUNCH if the launch is refused, else ATTN_OK. */
int attn_selftest_timeout(long long limit_ns, void* stream);

/* Diagnostic (no counterpart on the pages): exercises the work-counter takeover
 * check that attn_fwd, attn_fwd_window, attn_fwd_fp8 and attn_decode rely on, on a
 * counter reserved for it (no call of the library shares it).  Enqueues on `stream`:
 * a reset of that counter to launch generation 7; one CTA of generation 7 claiming
 * four times from 3 work units; a reset to generation 8; one CTA of generation 7
 * claiming once; one CTA of generation 8 claiming once.  `out` is a device array of
 * at least 6 ints; the claims land there in that order and read 0 1 2 -1 -1 1 (-1 =
 * no unit; generation 8 starts at 1 because the stale claim used up its unit 0), and
 * the following attn_get_device_status() returns ATTN_ERR_SCHED_CONFLICT (generation
 * 7 found the counter taken over).  Returns
 * ATTN_ERR_INVALID_ARG for NULL, ATTN_ERR_ALIGNMENT for a misaligned `out`,
 * ATTN_ERR_LAUNCH if a launch is refused, else ATTN_OK. */
int attn_selftest_sched(int* out, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
