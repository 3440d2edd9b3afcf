/*
 * fa.h - C ABI of the B200 (sm_100a) exact tiled attention library
 *        (libfa_b200.so).
 *
 * The operation.  Exact softmax attention, computed tile by tile so that
 * the N x N score matrix never reaches HBM ("FlashAttention:
 * Fast and Memory-Efficient Exact Attention with IO-Awareness",
 * opendecode.dev summary, section "The key idea"; "FlashAttention,
 * Decoded", gloss of abstract sentence 4 and "The Hardware Picture").  For
 * every batch b and head h, with row r and key c:
 *
 *   allowed(r,c) = (!causal || c <= r) && (kv_len == NULL || c < L_b)
 *                  && (block_mask == NULL || block_mask[(r/128)*nt + c/128] != 0)
 *   with L_b = kv_len[b] clamped into [0, N]
 *   S_rc  = scale * <Q_r, K_c>  (allowed), -inf (otherwise)
 *   P_rc  = exp(S_rc - LSE_r),  LSE_r = ln sum_c exp(S_rc)
 *   O_r   = sum_c P_rc V_c
 *
 * A row with no allowed key gets O_r = 0 and LSE_r = -inf.  The backward pass
 * recomputes S and P on chip from Q, K, V and LSE ("The Hardware Picture":
 * recomputation; opendecode.dev, "The key idea") and returns
 * dQ = scale * dS K, dK = scale * dS^T Q, dV = P^T dO, with
 * dS = P o (dO V^T - D) and D_r = sum_x dO_rx O_rx.
 *
 * Conventions for every entry point below.
 *  - Tensors Q, K, V, O, dO, dQ, dK, dV are bfloat16 (raw 16-bit patterns,
 *    type fa_bf16), contiguous [B][H][N][d] in device memory, base address
 *    16-byte aligned.  LSE is float32 [B][H][N] (natural log), 4-byte aligned.
 *  - d is 32, 64, 96, 128 or 256 (32 and 96 run on the 64- and 128-column
 *    kernels, whose loads read the missing columns as zeros and whose stores
 *    stop at d; the ordered dQ of fa_bwd_deterministic takes 64, 128 and 256;
 *    256 has kernels of its own, described at fa_bwd, and no dropout or
 *    packed variable-length form: those calls return FA_ERR_UNSUPPORTED_D).
 *    N is any length: tiles are 128 long, and when 128 does
 *    not divide N the last tile is partial.  B, H, N >= 0; if any is 0 the
 *    call does nothing and returns FA_OK.  B*H*N must be below 2^31.
 *  - scale is finite and > 0 (1/sqrt(d) is the usual choice).
 *  - block_mask (nullable) is uint8 [nt][nt] with nt = ceil(N/128), in device
 *    memory, row = query tile, column = key tile, nonzero = keep; all (b, h)
 *    share it; a last, partial tile's row and column cover its positions.
 *  - kv_len (nullable) is int32 [B] in device memory: keys c >= kv_len[b]
 *    are masked for every query of batch b.  Values must lie in [0, N];
 *    the kernels clamp values outside that range into it.
 *  - stream is a cudaStream_t (passed as void*; NULL = legacy default
 *    stream).  Work is enqueued asynchronously; the return value covers
 *    argument checks and launch errors only.  Device-side failures (a
 *    pipeline wait that timed out) are reported by fa_get_device_status.
 *  - The caller owns every buffer.  fa_fwd allocates nothing.  fa_bwd uses
 *    only the caller's workspace.  Nothing is freed by the library.
 *  - On any nonzero return, nothing was launched and no output was touched.
 *  - Each call makes the device that holds q current and launches there.
 *    Calls may come from several host threads and target several devices
 *    of one process; the library's per-device set-up (the kernels' shared
 *    memory opt-in, the SM count) is made once per device.
 *  - Kernels are launched with programmatic stream serialization: each may
 *    be scheduled while the previous kernel in the stream is finishing and
 *    waits, before it touches global memory, until that kernel's writes are
 *    visible.  Stream order is kept; a caller's own kernel that follows on
 *    the stream starts early only if it was launched that way itself.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t fa_bf16; /* bfloat16 bit pattern */

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = -1,           /* a required pointer is NULL */
    FA_ERR_ALIGN = -2,          /* a pointer breaks its alignment rule */
    FA_ERR_SHAPE = -3,          /* negative size, or B*H*N >= 2^31 */
    FA_ERR_UNSUPPORTED_D = -4,  /* d not in {32, 64, 96, 128, 256} ({64, 128, 256} for the
                                   ordered dQ; 256 with dropout or packed batches) */
    FA_ERR_WORKSPACE = -5,      /* workspace NULL or smaller than fa_bwd_workspace_size */
    FA_ERR_CUDA = -6,           /* a CUDA runtime/driver call failed */
    FA_ERR_TIMEOUT = -7,        /* a device pipeline wait gave up (fa_get_device_status) */
    FA_ERR_ARG = -8,            /* scale not finite or not > 0, phase not in 0..3, or
                                   p_drop outside [0, 1) */
    FA_ERR_SCRATCH_LIMIT = -9   /* fa_bwd_noalloc: the shape needs more scratch than
                                   FA_BWD_NOALLOC_SCRATCH_BYTES */
} fa_status;

/*
 * Forward pass: writes O and LSE.  One persistent launch; each CTA takes
 * (b, h, pair of 128-row query tiles) work units and streams the key/value
 * tiles that hold at least one allowed entry (causal, key-padding and
 * block-sparse tile skipping), with the online softmax (running row max and
 * row sum, partial output rescaled as tiles arrive; opendecode.dev, "The
 * key idea").
 */
int fa_fwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
           int B, int H, int N, int d, float scale, int causal,
           const uint8_t* block_mask, const int32_t* kv_len, void* stream);

/*
 * fa_fwd plus a record of the tiles it computed: visited (device, uint8
 * [B][H][nt][nt] (nt = ceil(N/128)), zeroed by the caller) gets 1 at [b][h][i][j] for
 * every (query tile i, key tile j) whose scores the kernel formed.  Same
 * kernel as fa_fwd; intended for tests of the tile-skip logic.
 */
int fa_fwd_traced(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                  int B, int H, int N, int d, float scale, int causal,
                  const uint8_t* block_mask, const int32_t* kv_len, uint8_t* visited,
                  void* stream);

/*
 * Bytes of device workspace fa_bwd needs: 4*B*H*Np (D) + 4*B*H*Np (LSE in
 * base 2) + 4*B*H*N*d (float32 dQ accumulator; none at d = 256) + 256 (the
 * counter from which the main kernel's CTAs take work units), each region
 * 256-byte aligned, where Np is N rounded up to a multiple of 128.
 * Returns 0 for an empty or invalid shape.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward pass: from Q, K, V, O, LSE (as written by fa_fwd with the same
 * mask arguments) and dO, writes dQ, dK, dV.  Three launches on `stream`:
 * a preprocess kernel (D = rowsum(dO o O), zero the dQ accumulator), the
 * main kernel (one CTA per (b, h, 128-key tile): recompute S and P,
 * accumulate dK and dV on chip, add dQ partials into the float32
 * accumulator), and a kernel that writes dQ = bf16(scale * accumulator).
 * At d = 256 a 128-key tile's float32 dK and dV would fill tensor memory, so
 * the work after the preprocess kernel is three passes instead, each
 * recomputing the score tile it needs: dK per key tile, dV per key tile, and
 * dQ per query tile summed on chip in a fixed order (no accumulator in the
 * workspace; the result is bitwise reproducible).
 * workspace must be 256-byte aligned and hold fa_bwd_workspace_size bytes;
 * its contents on entry do not matter and on exit are unspecified.  Calls
 * that share a workspace must not overlap on the device.
 */
int fa_bwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
           const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
           int B, int H, int N, int d, float scale, int causal,
           const uint8_t* block_mask, const int32_t* kv_len,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd plus a record of the tiles the main kernel computed: visited
 * (device, uint8 [B][H][nt][nt] (nt = ceil(N/128)), zeroed by the caller) gets 1 at
 * [b][h][i][j] for every (query tile i, key tile j) it recomputed.
 */
int fa_bwd_traced(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                  const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                  int B, int H, int N, int d, float scale, int causal,
                  const uint8_t* block_mask, const int32_t* kv_len,
                  void* workspace, size_t workspace_bytes, uint8_t* visited, void* stream);

/*
 * One launch of fa_bwd or fa_bwd_deterministic, for callers that schedule or
 * time them separately: phase 0 = preprocess (D, base-2 LSE, zeroed dQ
 * accumulator and work-unit counter in the workspace), 1 = main kernel (dK,
 * dV; dQ partials into the accumulator; takes its work units from the
 * counter, so each phase 1 needs a phase 0 before it), 2 = dQ = bf16(scale *
 * accumulator), 3 = dQ by the ordered kernel of fa_bwd_deterministic (reads
 * only what phase 0 wrote).  At d = 256: phase 1 = the dK and dV passes,
 * phases 2 and 3 = the dQ pass.  Arguments as for
 * fa_bwd.  Calling phases 0, 1, 2 in order on one stream with the same
 * arguments and workspace is exactly fa_bwd, and 0, 1, 3 is exactly
 * fa_bwd_deterministic; a phase reads what the earlier phases left in the
 * workspace.
 */
int fa_bwd_phase(int phase, const fa_bf16* q, const fa_bf16* k, const fa_bf16* v,
                 const fa_bf16* o, const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk,
                 fa_bf16* dv, int B, int H, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, const int32_t* kv_len, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * fa_bwd with a bitwise-reproducible result: the same arguments and
 * workspace, the same outputs within rounding, and on every run on the same
 * device the same bits.  fa_bwd's dQ sums the key tiles' contributions with
 * reduce-adds whose order varies between runs; here one CTA owns each query
 * tile and adds its visited key tiles' dS K_j products in increasing j, on
 * chip (recomputing S, P and dP for the purpose), and writes dQ once.  The
 * backward pass of the pages recomputes the score tiles instead of storing
 * them ("FlashAttention, Decoded", "The Hardware Picture"); the order of the
 * sums is this library's choice.  Costs about 60% more tensor-core work than
 * fa_bwd.  Three launches: preprocess, main kernel (dK, dV), ordered dQ.
 */
int fa_bwd_deterministic(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                         const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk,
                         fa_bf16* dv, int B, int H, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, const int32_t* kv_len, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Forward and backward passes with dropout on the attention probabilities,
 * fused into the same kernels.  Standard attention runs masking, softmax and
 * dropout as separate memory-bound passes over the N x N matrix ("FlashAttention:
 * A Novel Attention Algorithm with IO Awareness, Fast and Memory-Efficient",
 * "Standard Attention Algorithm", the GPT-2 time breakdown); here the keep
 * mask is drawn on chip and never stored.  The backward pass draws the same
 * mask again from the same counters.
 *
 *   O_r  = sum_c P_rc Z_rc V_c,  Z_rc = w * keep(b*H + h, r, c) with
 *   w = 65536 / (65536 - t),  t = floor(p_drop * 65536) (single precision,
 *   where that product is exact), keep = (16-bit draw >= t).
 *   The draw for (head index bh = b*H + h, query r, key c) is value c % 8 of
 *   Philox-4x32-10 (Salmon et al., SC 2011) with counter
 *   (c / 8, r, bh, offset) and key (seed low 32 bits, seed high 32 bits):
 *   value k is the low 16 bits of output word k/2 for even k, the high 16
 *   bits for odd k.
 *   LSE is the softmax's and does not depend on the mask.  The backward pass
 *   returns the gradients of that O: dV = (P o Z)^T dO,
 *   dS = P o (Z o (dO V^T) - D) with D_r = sum_x dO_rx O_rx (O the dropped
 *   output), dQ = scale * dS K, dK = scale * dS^T Q.
 *
 * p_drop must lie in [0, 1) (FA_ERR_ARG otherwise); p_drop = 0 keeps every
 * entry and gives fa_fwd's and fa_bwd's results.  Pass the same p_drop, seed
 * and offset to both passes; callers advance offset (or seed) between
 * layers or steps that must draw independent masks.  All other arguments,
 * layouts and error codes are those of fa_fwd and fa_bwd.  There is no
 * deterministic-dQ variant with dropout.
 */
int fa_fwd_dropout(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                   const int32_t* kv_len, float p_drop, uint64_t seed, uint32_t offset,
                   void* stream);

int fa_bwd_dropout(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                   const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                   const int32_t* kv_len, float p_drop, uint64_t seed, uint32_t offset,
                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Packed variable-length batches: B sequences of different lengths stored
 * token after token, with no padding.  Sequence b is tokens cu_seqlens[b] ..
 * cu_seqlens[b+1] - 1, and each sequence is its own attention problem (the
 * operation above with N = its length; causal masks are top-left aligned
 * within the sequence).
 *  - Q, K, V, O, dO, dQ, dK, dV: bfloat16 [T][H][d] (T = total_tokens =
 *    cu_seqlens[B]), 16-byte aligned; LSE: float32 [H][T].
 *  - cu_seqlens: int32 [B + 1] in device memory, 4-byte aligned, with
 *    cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] = T, and every length at
 *    most max_seqlen.  The kernels clamp each sequence into [0, T) and its
 *    length into [0, max_seqlen], so inconsistent values give wrong results
 *    for those sequences but never an access outside the tensors.
 *  - Host checks: B, H, max_seqlen, total_tokens >= 0 (FA_ERR_SHAPE);
 *    total_tokens <= B * max_seqlen (FA_ERR_SHAPE); B*H*max_seqlen < 2^31;
 *    cu_seqlens non-NULL (FA_ERR_NULL) and 4-byte aligned (FA_ERR_ALIGN); d,
 *    scale and p_drop as elsewhere.  If B, H, max_seqlen or total_tokens is 0
 *    the call does nothing and returns FA_OK.
 *  - p_drop, seed, offset: dropout as in fa_fwd_dropout (p_drop = 0: none);
 *    the draws number heads b*H + h and rows and keys within the sequence.
 *  - No block mask and no kv_len (a sequence's length is its key length).
 *  - fa_bwd_varlen's workspace: fa_bwd_workspace_size(B, H, max_seqlen, d)
 *    bytes, 256-byte aligned.
 * Work is scheduled on the grid of B x H x ceil(max_seqlen / 128) tiles;
 * tiles past a shorter sequence's end are skipped.
 */
int fa_fwd_varlen(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                  const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total_tokens, int d,
                  float scale, int causal, float p_drop, uint64_t seed, uint32_t offset,
                  void* stream);

int fa_bwd_varlen(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                  const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                  const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total_tokens, int d,
                  float scale, int causal, float p_drop, uint64_t seed, uint32_t offset,
                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * Self-test of the failure path every kernel relies on.  Each pipeline wait
 * in the kernels is bounded in time; when a wait gives up, the kernel records
 * a timeout in a device status word, winds down and exits, and
 * fa_get_device_status then returns FA_ERR_TIMEOUT (and clears the word).
 * This call launches one warp that waits on a shared-memory barrier for at
 * most limit_us microseconds (1 .. 2,000,000, else FA_ERR_ARG).  With
 * arrive = 0 nothing completes the barrier, so the wait must give up and
 * record the timeout; with arrive != 0 the warp arrives first and the wait
 * succeeds.  *result (device memory, int, 4-byte aligned) is set to 1 if the
 * wait succeeded, 0 if it gave up.  No fault, trap or unbounded wait is
 * involved: the kernel always ends, and the context stays usable.
 */
int fa_selftest_wait_timeout(int arrive, unsigned int limit_us, int* result, void* stream);

/*
 * Self-test of the softmax's exponential on the FMA pipe.  Part of the
 * exponentials 2^x of the forward and backward kernels are computed without
 * the special-function unit: x = n + f with n = round(x) and |f| <= 1/2, 2^f
 * as a degree-3 polynomial (the minimax fit for relative error, at most
 * 7.5e-5), and n added to the result's exponent field; x below -126 is taken
 * as -126.  This call writes y[i] = that function of x[i] for i < n
 * (pair = 0: the one-value form; pair != 0: the two-value form the kernels
 * run on packed pairs, which must give the same results).  x and y are
 * float32 arrays in device memory, 4-byte aligned.  n < 0 gives
 * FA_ERR_SHAPE; n = 0 does nothing.  Asynchronous on `stream`.
 */
int fa_selftest_ex2(const float* x, float* y, int n, int pair, void* stream);

/*
 * Size in bytes of the library's built-in backward scratch buffer (64 MiB),
 * used only by fa_bwd_noalloc.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * fa_bwd without a caller-provided workspace, for callers that cannot
 * allocate device memory themselves: code that runs where the host side owns
 * no device allocator (a plugin handed only input and output buffers by its
 * host application), or deployments that forbid device allocations after
 * start-up.  The method itself has no counterpart: it is an interface
 * convenience.
 *
 * Same arguments and results as fa_bwd, minus the workspace.  The scratch
 * (D, base-2 LSE and the float32 dQ accumulator) lives in one static device
 * array of FA_BWD_NOALLOC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library holds until the process exits.  The call allocates
 * and frees nothing.
 *  - Shapes whose scratch (fa_bwd_workspace_size) exceeds that size return
 *    FA_ERR_SCRATCH_LIMIT and launch nothing.  With d = 64 that admits
 *    B*H*N up to about 254K rows; with d = 128 about 129K rows.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current) and caches it; make
 *    that first call before any stream capture.  The cache is tied to the
 *    device's context: after cudaDeviceReset the next call looks the address
 *    up again (so make that call, too, outside a capture).
 *  - Every call on a device shares the one array.  Each call overwrites what
 *    it reads (the accumulator is zeroed by the call's first kernel), so the
 *    contents a previous call left behind do not matter, but calls whose
 *    kernels overlap on the device (two streams, or two host threads) race
 *    on the array and give wrong results: serialise them.
 */
int fa_bwd_noalloc(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                   const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                   int B, int H, int N, int d, float scale, int causal,
                   const uint8_t* block_mask, const int32_t* kv_len, void* stream);

/*
 * Synchronises `stream`, then returns FA_OK if no kernel of this library
 * has reported a device-side failure since the last call, FA_ERR_TIMEOUT
 * if a pipeline wait gave up (the kernel then skipped the rest of its work
 * and its outputs are incomplete), or FA_ERR_CUDA if synchronising failed.
 * Clears the recorded state.  The state is per process and per device, and
 * the call reads that of the calling thread's current device: the device of
 * the last entry point this thread called (each call makes q's device
 * current), so pass a stream of that device.
 */
int fa_get_device_status(void* stream);

/* Static, NUL-terminated description of a status code. */
const char* fa_status_string(int status);

/* Library version as major*10000 + minor*100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
