/*
 * fa.h -- C ABI of libfa.so: exact softmax attention, forward and backward,
 * computed tile by tile with the online-softmax state on NVIDIA B200 (sm_100a).
 *
 * What is computed (per batch b and query head h, kv head kh = h / (H / Hkv)):
 *   S = scale * Q K^T, masked;  P = softmax(S) row-wise;  O = P V
 * ("Flash attention and efficient attention", section "The Standard Attention
 * Problem"; the scale there is 1/sqrt(d_k) and is an argument here).  The N x N
 * matrices S and P are never written to device memory: only O and the per-row
 * logsumexp LSE are ("FlashAttention" guide page, section "Tiling through
 * SRAM").  The backward recomputes S and P per tile from Q, K, V and LSE
 * ("Flash attention and efficient attention", section "Backward Pass:
 * Recomputation") and returns the gradients of L = sum(dO * O).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  Layouts   all tensors contiguous, row-major, head dim d fastest:
 *              q, o, dout, dq      [B, H,   N, d]
 *              k, v, dk, dv        [B, Hkv, N, d]
 *              lse                 [B, H,   N]   fp32, natural log of
 *                                  sum_j exp(S_ij) over the allowed keys
 *  dtype     FA_BF16: q/k/v/o/dout/dq/dk/dv are bfloat16 (fp32 accumulation);
 *            FA_FP32: they are float.  lse and the workspace are always float.
 *  Masks     causal != 0 keeps keys j <= i; window >= 0 keeps |i - j| <= window
 *            (half-width: the pages' "w = 3, itself plus one neighbour each
 *            side" is window = 1); window = -1 disables the band; both may be
 *            combined (i - window <= j <= i).
 *  Sizes     B, H, Hkv, N >= 1; H % Hkv == 0; d in {64, 128};
 *            scale finite and > 0.
 *  Pointers  device pointers (cudaMalloc'd or equivalent), 16-byte aligned;
 *            outputs must not alias inputs (not checked).  The caller owns all
 *            memory; the library allocates no device memory.
 *  stream    a cudaStream_t passed as void*; NULL means the legacy default
 *            stream.  Every call only enqueues work and returns without
 *            synchronising; results are ready when the stream reaches them.
 *            The kernels run on the current device (cudaSetDevice), which must
 *            be the stream's device and own every pointer; a stream of another
 *            device is rejected with FA_ERR_INVALID_ARG.
 *  Errors    argument errors are detected on the host before anything is
 *            enqueued and leave all buffers untouched; a failed launch returns
 *            FA_ERR_CUDA.  A device-side bounded wait that gives up (after about
 *            two seconds) records FA_ERR_TIMEOUT in a device status word that
 *            fa_last_device_status() reports.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null pointer, size < 1, H % Hkv != 0, bad scale/window/dtype */
  FA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. d not in {64, 128}) */
  FA_ERR_MISALIGNED = 3,  /* a pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,   /* workspace pointer null or ws_bytes too small */
  FA_ERR_CUDA = 5,        /* a CUDA runtime/driver call or a launch failed */
  FA_ERR_TIMEOUT = 6      /* a device-side bounded wait gave up */
} fa_status;

typedef enum fa_dtype { FA_BF16 = 0, FA_FP32 = 1 } fa_dtype;

/*
 * Forward: o = softmax(scale * q k^T, masked) v and lse (see above).
 * The online-softmax recurrence (running max m, running sum l, rescaled
 * unnormalised accumulator) is the one of "Flash attention and efficient
 * attention", section "Derivation: Incremental Softmax", Steps 1-3, applied
 * block after block of keys (the page states that the two-block merge extends
 * to any number of blocks).
 * Writes o [B,H,N,d] and lse [B,H,N]; reads q, k, v.  Deterministic.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int Hkv, int N, int d, float scale, int causal, int window,
                 fa_dtype dtype, void* stream);

/*
 * Split-KV forward: the same result as fa_fwd (o, lse), computed with the key
 * range of every 256-row query block cut into num_splits contiguous chunks that
 * run as separate CTAs.  Each chunk leaves its partial online-softmax state --
 * running maximum m, sums l (and l of the bf16-rounded weights), unnormalised
 * accumulator O~ -- in `workspace`; a second kernel merges them with the
 * block-merge identity of "Flash attention and efficient attention",
 * "Derivation: Incremental Softmax", Step 3, which the page extends to any
 * number of blocks.  More CTAs for the same work: for small B*H with long N.
 * bf16 only (FA_ERR_UNSUPPORTED for FA_FP32); 1 <= num_splits <= 16
 * (FA_ERR_INVALID_ARG otherwise); workspace: caller-owned device memory of at
 * least fa_fwd_splitkv_workspace_size() bytes, 16-byte aligned, contents
 * irrelevant on entry.  Results are not bitwise equal to fa_fwd's (different
 * summation order) and are deterministic.
 */
fa_status fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                         int N, int d, float scale, int causal, int window, int num_splits, void* workspace,
                         size_t ws_bytes, fa_dtype dtype, void* stream);

/* Workspace bytes fa_fwd_splitkv needs (0 for sizes it would reject). */
size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits);

/*
 * Decode: Nq <= Nk queries against Nk keys, forward only.  q, o [B, H, Nq, d],
 * k, v [B, Hkv, Nk, d], lse [B, H, Nq], all contiguous.  The queries are the
 * newest Nq tokens of a length-Nk sequence: query row i sits at position
 * Nk - Nq + i, and the causal / window predicate applies to that position
 * ("FlashAttention" guide page, "Key takeaways": generating tokens calls for
 * its own kernel mapping of the same computation).  With Nq == Nk this is fa_fwd.  The
 * key range of every query tile is cut into num_splits chunks processed by
 * separate CTAs, whose partial online-softmax states are merged on the device
 * exactly as in fa_fwd_splitkv -- what keeps a single short query tile from
 * running on one SM.  The H / Hkv query heads that share a kv head are
 * processed together (their g * Nq rows are adjacent in q and o), so each K/V
 * tile is read once per kv head, not once per query head.  workspace: at least
 * fa_fwd_decode_workspace_size(B, H, Hkv, Nq, d, num_splits) bytes, 16-byte
 * aligned.  bf16 only (FA_ERR_UNSUPPORTED otherwise); FA_ERR_INVALID_ARG for
 * Nq < 1, Nk < Nq or num_splits outside [1, 16]; other errors as fa_fwd.
 */
size_t fa_fwd_decode_workspace_size(int B, int H, int Hkv, int Nq, int d, int num_splits);
fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int Nq, int Nk, int d, float scale, int causal, int window, int num_splits, void* workspace,
                        size_t ws_bytes, fa_dtype dtype, void* stream);

/*
 * Block-sparse forward and backward: as fa_fwd / fa_bwd with an extra 0/1 mask
 * over 128 x 128 blocks of the score matrix; a key is allowed only if the
 * causal / window predicate allows it AND its block is on.  Block sparsity is
 * named on the "FlashAttention paper" page ("What it does not claim") as a
 * separate extension of the same tiled algorithm; switched-off blocks are never
 * loaded or multiplied.
 *  block_mask        device pointer, unsigned char, nb x nb per query head
 *                    (nb = ceil(N / 128)), row = query block, column = key block;
 *                    any nonzero byte means "on".
 *  mask_head_stride  elements between consecutive query heads' masks
 *                    (head index b * H + h); 0 = one mask for every head.
 * Rows left with no allowed key get O = 0, LSE = -inf and zero gradients.
 * Errors as fa_fwd / fa_bwd, plus FA_ERR_INVALID_ARG for a null block_mask or a
 * negative stride.  fa_bwd_workspace_size() applies unchanged.
 */
fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                             int Hkv, int N, int d, float scale, int causal, int window,
                             const unsigned char* block_mask, long long mask_head_stride, fa_dtype dtype,
                             void* stream);
fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                             int H, int Hkv, int N, int d, float scale, int causal, int window,
                             const unsigned char* block_mask, long long mask_head_stride, fa_dtype dtype,
                             void* stream);

/*
 * Padded variable lengths: as fa_fwd / fa_bwd on the same [B, H, N, d]
 * (and [B, Hkv, N, d]) layouts, where batch entry b holds only seqlens[b] valid
 * tokens at the start of its rows ("FlashAttention" guide page, "Tiling through
 * SRAM": padding only alters how the tiles are laid out, not what is computed).  Keys at positions >=
 * seqlens[b] are never attended to; query rows >= seqlens[b] get O = 0,
 * LSE = -inf and zero dQ; key rows >= seqlens[b] get zero dK, dV.  Whatever the
 * padding rows hold has no effect.  seqlens: device pointer to B int32 values,
 * each clamped to [0, N] on the device; FA_ERR_INVALID_ARG if null.  Other
 * arguments and errors as fa_fwd / fa_bwd.
 */
fa_status fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Hkv,
                        int N, int d, float scale, int causal, int window, const int* seqlens, fa_dtype dtype,
                        void* stream);
fa_status fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int H,
                        int Hkv, int N, int d, float scale, int causal, int window, const int* seqlens,
                        fa_dtype dtype, void* stream);

/*
 * Strided layouts: as fa_fwd_varlen / fa_bwd_varlen (seqlens may be NULL: every
 * batch entry then has N valid rows), but each tensor argument may have any
 * layout whose head dimension d is contiguous -- e.g. [B, N, H, d] ("BSHD",
 * tokens outer, heads inner), a slice of a longer buffer, or rows with a
 * padded pitch.  The same rule and outputs as fa_fwd / fa_bwd ("FlashAttention"
 * guide page, "Tiling through SRAM": the layout only changes how tiles are
 * addressed, and the tile schedule is the same).  lse stays [B, H, N]
 * contiguous fp32.
 *
 * strides: host pointer to 4 (fwd: q, k, v, o) or 8 (bwd: q, k, v, o, dout, dq,
 * dk, dv) fa_strides, in ELEMENTS: element (b, h, n, c) of a tensor is at
 * b * batch + h * head + n * row + c.  The contiguous [B, H, N, d] layout is
 * {H*N*d, N*d, d}; a [B, N, H, d] buffer seen as [B, H, N, d] is {N*H*d, d, H*d}.
 * Rules (FA_ERR_INVALID_ARG unless noted): every stride > 0 and < 2^40 bytes;
 * every stride times the element size a multiple of 16 bytes
 * (FA_ERR_MISALIGNED); the stride of an axis of extent 1 (B == 1, or a single
 * head) is ignored; an output layout (o, dq, dk, dv) must be one-to-one -- with
 * its axes sorted by stride, each stride at least the span of the axes inside
 * it (d for the innermost).  Inputs may overlap each other; outputs must not
 * overlap inputs or each other (not checked).  Elements of an output buffer
 * that no (b, h, n, c) maps to are never written.  Other arguments, errors and
 * fa_bwd_workspace_size() as fa_fwd / fa_bwd.
 */
typedef struct {
  long long batch, head, row; /* element strides; d is contiguous */
} fa_strides;
fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                         const fa_strides* strides, int B, int H, int Hkv, int N, int d, float scale, int causal,
                         int window, const int* seqlens, fa_dtype dtype, void* stream);
fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, const fa_strides* strides, void* workspace,
                         size_t ws_bytes, int B, int H, int Hkv, int N, int d, float scale, int causal, int window,
                         const int* seqlens, fa_dtype dtype, void* stream);

/*
 * Packed variable lengths: B sequences concatenated along the token axis, no
 * padding.  cu_seqlens: HOST pointer to B + 1 non-decreasing int32 offsets
 * with cu_seqlens[0] = 0 (validated, and used to size the launch);
 * cu_seqlens_dev: DEVICE pointer (16-byte aligned) to the same B + 1 values,
 * read by the kernels, so it must stay unchanged until the stream has run the
 * call (the fp32 path reads only the host copy and accepts NULL here; the
 * kernels clamp every offset to [0, T], so differing copies give wrong values,
 * never an access outside the tensors).  Sequence b occupies token rows
 * [cu_seqlens[b], cu_seqlens[b+1]) of
 *   q, o, dout, dq   [T, H, d]     (T = cu_seqlens[B], d contiguous)
 *   k, v, dk, dv     [T, Hkv, d]
 *   lse              float; sequence b's [H, len_b] block starts at element
 *                    H * cu_seqlens[b]
 * Each sequence is its own attention problem (causal / window relative to its
 * first token; "FlashAttention" guide page, "Tiling through SRAM": padding and
 * lengths only alter how the tiles are laid out, not what is computed).  bf16:
 * one launch of each kernel covers every sequence; tiles start at each
 * sequence's first row, and output rows are written only up to its end.  fp32:
 * one launch per sequence (empty sequences launch nothing).  fa_bwd_packed's
 * workspace: at least fa_bwd_packed_workspace_size(cu_seqlens, B, H, d, dtype)
 * bytes -- for bf16 every sequence's rows padded to whole 128-row tiles plus
 * 128 rows per sequence, per head; for fp32 the longest sequence's (reused
 * sequence after sequence, in stream order).  Errors: FA_ERR_INVALID_ARG for a
 * null or (bf16) missing / misaligned device offsets pointer, B < 1,
 * cu_seqlens[0] != 0, decreasing offsets or T + 128 (B + 1) >= 2^30 (bf16);
 * otherwise as fa_fwd / fa_bwd (with N the longest sequence).
 */
fa_status fa_fwd_packed(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens,
                        const int* cu_seqlens_dev, int B, int H, int Hkv, int d, float scale, int causal, int window,
                        fa_dtype dtype, void* stream);
size_t fa_bwd_packed_workspace_size(const int* cu_seqlens, int B, int H, int d, fa_dtype dtype);
fa_status fa_bwd_packed(const void* q, const void* k, const void* v, const void* o, const void* dout,
                        const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens,
                        const int* cu_seqlens_dev, void* workspace, size_t ws_bytes, int B, int H, int Hkv, int d,
                        float scale, int causal, int window, fa_dtype dtype, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for these sizes (fp32 row terms
 * D_i = sum_k dO_ik O_ik, prescaled LSE, and for bf16 a float dQ accumulator).
 * Returns 0 for sizes fa_bwd would reject.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d, fa_dtype dtype);

/*
 * Backward of fa_fwd for the loss L = sum(dout * o): writes dq [B,H,N,d],
 * dk and dv [B,Hkv,N,d].  Reads q, k, v, o, dout and the lse that fa_fwd wrote
 * for the same inputs; recomputes S and P per tile ("Flash attention and
 * efficient attention", "Backward Pass: Recomputation").  The gradients of a
 * kv head sum over its H / Hkv query heads.  workspace: caller-owned device
 * memory of at least fa_bwd_workspace_size() bytes, 16-byte aligned; its
 * contents on entry do not matter and are garbage on return.  dk, dv, o and
 * lse are deterministic; dq (bf16 path) adds the tile contributions in L2 in
 * whatever order they arrive (TMA bulk reduce-adds), so its last bits may vary
 * from run to run.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                 int B, int H, int Hkv, int N, int d, float scale, int causal, int window,
                 fa_dtype dtype, void* stream);

/*
 * Size of the built-in scratch buffer used by fa_bwd_noalloc (16 MiB).
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)

/*
 * fa_bwd without a caller-supplied workspace.  (The pages have no counterpart:
 * this exists for callers, not for the method.)  Some callers cannot allocate
 * device memory at all -- a plugin running inside a host application that owns
 * every device allocation and hands the plugin no allocator, or a latency-bound
 * loop in which a cudaMalloc, which may synchronise the device, is forbidden.
 * They still pass q, k, v, o, dout, lse and the dq/dk/dv outputs exactly as for
 * fa_bwd; the scratch fa_bwd would take from `workspace` comes instead from one
 * file-scope device array of FA_BWD_NOALLOC_SCRATCH_BYTES bytes that every GPU
 * which loads libfa.so holds until the process exits.  Nothing here calls
 * cudaMalloc, cudaFree or any allocating routine.
 *  - Limit: problems whose fa_bwd_workspace_size() exceeds
 *    FA_BWD_NOALLOC_SCRATCH_BYTES are rejected with FA_ERR_WORKSPACE before
 *    anything is enqueued (e.g. bf16, d = 128: B*H*ceil(N/128)*128 <= 32256).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make that
 *    first call before any stream capture.
 *  - All calls on a device share the one array and leave their contents in
 *    it (each call clears what must start at zero itself); calls that can
 *    overlap on the GPU -- different streams without ordering between them --
 *    race on it and must be serialised by the caller.
 * Other arguments, layouts and errors as fa_bwd.
 */
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout,
                         const float* lse, void* dq, void* dk, void* dv, int B, int H, int Hkv, int N, int d,
                         float scale, int causal, int window, fa_dtype dtype, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device status word:
 * FA_ERR_TIMEOUT if a kernel's bounded wait gave up since the last call,
 * FA_ERR_CUDA if the synchronisation itself failed, else FA_OK.
 */
fa_status fa_last_device_status(void* stream);

/*
 * Optional timing hook for benchmarks (off by default).  While both events are
 * non-NULL, every later fa_fwd / fa_bwd call records `start` on its stream just
 * before its main attention kernel and `stop` just after it (the forward
 * kernel; for fa_bwd the tile-recomputing kernel, not the row-term preprocess
 * or the dQ conversion).  Arguments are cudaEvent_t passed as void*; pass NULLs
 * to switch it off.  Process-wide and not thread-safe.
 */
void fa_set_timing_events(void* start, void* stop);

/*
 * Test hooks for the failure-detection path (not for production use; both are
 * process-wide, per device, and take effect for kernels launched afterwards).
 *
 * fa_debug_set_wait_limit: the limit, in nanoseconds, after which a kernel's
 *   wait for another role of its CTA (a tile load, a tensor-core product, a
 *   softmax step) gives up; 0 restores the default of about two seconds.  A
 *   CTA whose wait gives up records FA_ERR_TIMEOUT in the device status word,
 *   stops its other roles, waits (always with the default limit) for its own
 *   copies and tensor-core operations in flight, frees its tensor memory and
 *   returns; the outputs of that call are then undefined.
 * fa_debug_set_stall: while nonzero, the sm_100a kernels never issue their
 *   first tile load (K/V in the backward, Q in the forward), so every CTA's
 *   waits for it run out and the call reports FA_ERR_TIMEOUT through
 *   fa_last_device_status(); 0 restores normal operation.  The fp32 path has
 *   no waits and ignores it.
 * Both synchronise with the device (cudaMemcpyToSymbol on the legacy stream)
 * and return FA_ERR_CUDA if that fails.
 */
fa_status fa_debug_set_wait_limit(unsigned long long ns);
fa_status fa_debug_set_stall(int on);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(fa_status s);

/* Library ABI version (major * 100 + minor). */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
