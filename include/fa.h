/*
 * fa.h — C ABI of the B200 (sm_100a) exact attention library (libfa.so).
 *
 * The operation is exact scaled-dot-product attention as FlashAttention
 * computes it:
 *   S = scale * Q K^T, P = softmax(S) row by row, O = P V
 * ("FlashAttention" interview explainer, mstx.cn/posts/485, section 2.1,
 * standard attention; the 1/sqrt(d) scale as in the nanhubrain.csdn.net
 * FlashAttention essay, section 2). The forward streams K/V tiles past each
 * resident Q tile with the online-softmax recurrence (same explainer, section
 * 3.2) and writes only O and the per-row logsumexp. The backward recomputes P
 * from Q, K and the saved logsumexp instead of storing it ("FlashAttention"
 * concept card, lukebest.github.io, "反向：重算而非存储").
 *
 * Conventions shared by every entry point
 *   - Tensors q, k, v, o, dout, dq, dk, dv are contiguous [B, H, N, d] in the
 *     element type given by `dtype` (fp16 or bf16); lse is contiguous fp32
 *     [B, H, N]. All are DEVICE pointers, 16-byte aligned.
 *   - lse_i = ln sum_j exp(scale * q_i . k_j) over the keys row i may see
 *     (natural log, in the units of the scaled scores).
 *   - d must be 32, 64, 96 or 128, or 256 for the forward entry points
 *     (fa_fwd, fa_fwd_qk, fa_blocksparse_fwd, fa_fwd_splitkv; the backward,
 *     dropout and 8-bit entry points return FA_ERR_UNSUPPORTED for it). 32 and
 *     96 run in the 64 and 128 kernels with the missing columns zero-filled, at
 *     the cost of the padded width; 256 runs one query tile per CTA;
 *     N >= 1 (any value; ragged last tiles are handled); B, H >= 1 and
 *     B*H <= 65535.
 *   - causal != 0 masks key j > query i (top-left aligned; the essay's
 *     section 3.1 causal mask P_ij = 0 for j > i).
 *   - The caller owns all memory. The library allocates no device memory; the
 *     backward takes a caller-provided workspace of fa_bwd_workspace_size()
 *     bytes. Host-side tensor-map descriptors are built per call.
 *   - Every call is asynchronous on `stream` and never synchronises. Argument
 *     errors are reported before any launch; a failed launch returns
 *     FA_ERR_CUDA. Device-side time-outs (a wait that could not complete) are
 *     recorded in a device status word read by fa_device_status().
 *   - A row with no allowed key (possible only with a block mask) gets O = 0,
 *     lse = -inf and contributes zero gradients.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, non-positive size, bad dtype */
  FA_ERR_UNSUPPORTED = 2, /* valid but unsupported shape (head dimension, size limits) */
  FA_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  FA_ERR_TIMEOUT = 4      /* a device-side wait gave up (see fa_device_status) */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;

/* Human-readable name of a status code (static string). */
const char* fa_status_string(fa_status s);

/*
 * Forward. Writes o [B,H,N,d] (dtype) and lse [B,H,N] (fp32).
 * q, k, v are read only. softmax_scale is usually 1/sqrt(d).
 */
fa_status fa_fwd(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int N, int d, float softmax_scale, int causal, cudaStream_t stream);

/*
 * Bytes of device workspace fa_bwd / fa_blocksparse_bwd need for these sizes:
 * two fp32 row vectors [B,H,ceil(N/128)*128] (D = rowsum(dO o O) and lse in
 * log2 units). Linear in N. Returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward. Given the forward's inputs, its outputs o and lse, and the
 * incoming gradient dout = dL/dO, writes dq, dk, dv [B,H,N,d] (dtype):
 *   D = rowsum(dO o O), P = exp(scale*Q K^T - lse), dV = P^T dO,
 *   dP = dO V^T, dS = P o (dP - D), dQ = scale*dS K, dK = scale*dS^T Q.
 * P is recomputed from Q, K and lse rather than stored ("FlashAttention"
 * concept card, lukebest.github.io, "反向：重算而非存储"). dS is the softmax
 * Jacobian applied to dP: the softmax gradient printed in the cloud.baidu.com
 * explainer ("梯度计算优化") is dimensionally inconsistent, so the textbook
 * form above is used; D_i = rowsum(P o dP)_i equals rowsum(dO o O)_i.
 * workspace: device buffer of at least fa_bwd_workspace_size() bytes, 256-byte
 * aligned; its contents on entry do not matter and are overwritten.
 */
fa_status fa_bwd(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int N, int d,
                 float softmax_scale, int causal, cudaStream_t stream);

/*
 * fa_bwd without a workspace argument, for callers that cannot allocate device
 * memory (a host application that owns every byte of device memory and gives
 * this library no allocator, or a latency-critical loop where cudaMalloc is
 * not allowed). The pages describe no such variant; it has no counterpart
 * there. Arguments and results are those of fa_bwd (without block mask).
 * Scratch: a fixed array of FA_BWD_NOALLOC_SCRATCH_BYTES bytes in the
 * library's static device memory, held by every GPU that loads the library
 * until the process exits. If fa_bwd_workspace_size(B, H, N, d) exceeds it the
 * call returns FA_ERR_UNSUPPORTED and launches nothing. All calls on a device
 * share that array: calls whose kernels may overlap on the GPU race and must be
 * ordered by the caller. Nothing in it needs to start at zero: every call's
 * first kernel rewrites all the entries (D and lse in log2 units) its second
 * kernel reads. Every other limit is that of fa_bwd. The first call on a device
 * looks up the array's device address (cudaGetSymbolAddress) and caches it;
 * make that first call before any stream capture. Allocates nothing.
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (32u << 20)
fa_status fa_bwd_noalloc(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                         const float* lse, const void* dout, void* dq, void* dk, void* dv, int B, int H, int N,
                         int d, float softmax_scale, int causal, cudaStream_t stream);

/*
 * Block-sparse forward ("FlashAttention" concept card, "Block-Sparse
 * FlashAttention": a fixed block mask whose zero blocks are skipped).
 * block_mask: DEVICE pointer to uint8 [N/128][N/128], row-major, shared by all
 * (b, h); entry (I, J) != 0 lets query tile I (rows 128I..128I+127) attend to
 * key tile J. Zero tiles are never loaded. Composes with `causal` by AND.
 * Requires N % 128 == 0 and N/128 <= 2048 (else FA_ERR_UNSUPPORTED).
 */
fa_status fa_blocksparse_fwd(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream);

/* Block-sparse backward; arguments as fa_bwd plus block_mask as in fa_blocksparse_fwd. */
fa_status fa_blocksparse_bwd(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream);

/*
 * Forward with Nq query rows and Nk key/value rows (a query block that is the
 * last Nq positions of a longer key sequence, cross-attention, decoding). The
 * pages treat the square case; this generalises the same computation:
 * q, o [B,H,Nq,d]; k, v [B,H,Nk,d]; lse [B,H,Nq]. The causal mask is
 * bottom-right aligned: query i attends to key j iff j <= i + Nk - Nq (for
 * Nq = Nk the rule j <= i). A query row with no key gets O = 0, lse = -inf.
 * block_mask may be NULL; otherwise it is a DEVICE uint8 [Nq/128][Nk/128] as
 * in fa_blocksparse_fwd and needs Nq, Nk multiples of 128 (at most 2048 tiles
 * each). With Nq = Nk this computes exactly what fa_fwd / fa_blocksparse_fwd do.
 * Errors, ownership and stream semantics as fa_fwd.
 */
fa_status fa_fwd_qk(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                    cudaStream_t stream);

/*
 * Backward of fa_fwd_qk: dq [B,H,Nq,d]; dk, dv [B,H,Nk,d]; o, dout [B,H,Nq,d];
 * workspace of at least fa_bwd_workspace_size(B, H, Nq, d) bytes (256-byte
 * aligned). Rows without keys contribute nothing. Otherwise as fa_bwd.
 */
fa_status fa_bwd_qk(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk,
                    int d, float softmax_scale, int causal, const uint8_t* block_mask, cudaStream_t stream);

/*
 * Split-KV forward (FlashDecoding, the "FlashAttention" concept card's lineage
 * table: partial softmax per key range, then a synchronising merge). Computes
 * exactly what fa_fwd_qk computes, with more parallelism when B*H*ceil(Nq/128)
 * is small next to the GPU (decoding: a few query rows against a long key
 * sequence). The Nk keys are cut into n_splits consecutive ranges of whole
 * 128-key tiles: range s holds key tiles [s*T/n_splits, (s+1)*T/n_splits),
 * T = ceil(Nk/128). Step 1 computes, for every query row and range, the
 * softmax-weighted mean of that range's values, O_s (fp32), and the log of its
 * exp-sum, lse_s (fp32, -inf if the row has no allowed key in the range); step 2
 * merges them: lse = log sum_s exp(lse_s), O = sum_s exp(lse_s - lse) O_s (the
 * online-softmax update of the interview explainer, section 3.2, applied to
 * whole ranges).
 * Arguments as fa_fwd_qk (q, o [B,H,Nq,d]; k, v [B,H,Nk,d]; lse [B,H,Nq];
 * bottom-right causal; optional block_mask [Nq/128][Nk/128]), plus:
 *   n_splits  1 <= n_splits <= ceil(Nk/128) (else FA_ERR_INVALID_ARG);
 *             fa_fwd_splitkv_splits() suggests one.
 *   workspace DEVICE buffer of fa_fwd_splitkv_workspace_size() bytes, 256-byte
 *             aligned, owned by the caller; on return (after the stream
 *             completes) it holds the partials: O_s as fp32
 *             [n_splits][B*H][Nq][d] at offset 0, then lse_s as fp32
 *             [n_splits][B*H][Nq] at the next 256-byte boundary after O_s.
 * Two launches on `stream`; asynchronous, allocates nothing. With Nq <= 4
 * (decoding) step 1 runs on the CUDA cores, which read each range's K and V
 * once; larger Nq use the tensor-core forward. The partials are the same.
 */
size_t fa_fwd_splitkv_workspace_size(int B, int H, int Nq, int d, int n_splits);
int fa_fwd_splitkv_splits(int B, int H, int Nq, int Nk);
fa_status fa_fwd_splitkv(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                         int n_splits, void* workspace, cudaStream_t stream);

/*
 * Attention with dropout on the probabilities, fused in the same kernels
 * ("FlashAttention" concept card, 算法要点 "Kernel fusion": QK^T -> softmax
 * (+ mask / dropout) -> PV). O = (P o Z) V, with P the softmax of the scaled,
 * masked scores (lse is that of P) and Z the dropout keep decisions: element
 * (i, j) of head bh = b*H + h is kept iff its draw u >= t, t = floor(256 p + 1/2),
 * and a kept entry is 256 / (256 - t) (so p is used rounded to t/256). The
 * draws come from Philox4x32-10 (Salmon et al., SC'11): one block per 4 x 4
 * block of (query row, key), counter (j >> 2, i >> 2, bh, 0), key (seed low
 * 32 bits, seed high 32 bits); output word (i & 3) holds row i's draws, byte
 * (j & 3) of it, least significant first, is u. The backward draws them again
 * from the same seed (nothing is stored) and computes, through O = (P o Z) V:
 * dV = (P o Z)^T dO, dP = (dO V^T) o Z, dS = P o (dP - D) with
 * D = rowsum(dO o O), dQ = scale dS K, dK = scale dS^T Q.
 * Arguments as fa_fwd_qk / fa_bwd_qk, plus p_drop in [0, 1) (else
 * FA_ERR_INVALID_ARG; p_drop = 0 is exactly fa_fwd_qk / fa_bwd_qk) and the
 * 64-bit seed; fa_bwd_dropout must get the forward's p_drop and seed.
 */
fa_status fa_fwd_dropout(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse, int B,
                         int H, int Nq, int Nk, int d, float softmax_scale, int causal, const uint8_t* block_mask,
                         float p_drop, unsigned long long seed, cudaStream_t stream);
fa_status fa_bwd_dropout(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace, int B, int H, int Nq, int Nk,
                         int d, float softmax_scale, int causal, const uint8_t* block_mask, float p_drop,
                         unsigned long long seed, cudaStream_t stream);

/*
 * 8-bit forward (the FP8 variant the "FlashAttention" concept card's lineage
 * table lists for FlashAttention-3). q8 [B,H,Nq,128], k8 and v8 [B,H,Nk,128]
 * are DEVICE arrays of e4m3 values (1 sign, 4 exponent bits with bias 7, 3
 * mantissa bits; one byte each); the tensors attended are q_scale * q8,
 * k_scale * k8, v_scale * v8 (per-tensor scales > 0). Writes O [B,H,Nq,128] as
 * bf16 and lse [B,H,Nq] (fp32) of exact attention on those tensors, with the
 * masks of fa_fwd_qk (bottom-right causal, optional block_mask). S = Q K^T runs
 * on the stored e4m3 values (kind::f8f6f4 MMAs, fp32 accumulation; the scales
 * join the softmax scale); V is widened to bf16 on chip and P V runs in bf16.
 * d must be 128 (else FA_ERR_UNSUPPORTED); scales must be finite and > 0 (else
 * FA_ERR_INVALID_ARG). Otherwise as fa_fwd_qk.
 */
fa_status fa_fwd_fp8(const void* q8, const void* k8, const void* v8, float q_scale, float k_scale, float v_scale,
                     void* o, float* lse, int B, int H, int Nq, int Nk, int d, float softmax_scale, int causal,
                     const uint8_t* block_mask, cudaStream_t stream);

/*
 * Debug: the dropout draws u (uint8) of every (head, query row, key) for
 * B*H heads, Nq query rows, Nk keys, written to two DEVICE buffers of
 * B*H*Nq*Nk bytes, [bh][i][j]: row_major through the generator path of the
 * forward and query-stationary backward (a thread per query row), col_major
 * through that of the key-stationary backward (a thread per key). Both equal
 * the layout described at fa_fwd_dropout.
 */
fa_status fa_debug_dropout_draws(int B, int H, int Nq, int Nk, unsigned long long seed, uint8_t* row_major,
                                 uint8_t* col_major, cudaStream_t stream);

/*
 * Debug: the forward / backward with a record of the tiles each CTA loaded.
 * trace: DEVICE int32 buffer of fa_*_trace_size() entries; each record is a
 * count followed by entries (tile index) | (flags << 16).
 * Forward: T_kv = ceil(N/128) key tiles; CTA c covers query tiles 2p and 2p+1
 * (p = c % n_pairs, n_pairs = ceil(T_kv/2)) of head c / n_pairs; its record of
 * T_kv + 1 entries starts at c * (T_kv + 1); flags bit q = the key tile is used
 * by query tile 2p+q.
 * Backward: key-stationary CTA (head h, key tile j) lists the query tiles of
 * fa_bwd_row_tile(d) rows it visits, record of T_q + 1 entries at
 * (h * T_kv + j) * (T_q + 1), T_q = ceil(N / fa_bwd_row_tile(d)); after all of
 * those, query-stationary CTA (head h, 128-row query tile i) lists the key
 * tiles it visits, record of T_kv + 1 entries at
 * B*H*T_kv*(T_q + 1) + (h * T_kv + i) * (T_kv + 1). Backward flags = 1.
 */
size_t fa_fwd_trace_size(int B, int H, int N);
size_t fa_bwd_trace_size(int B, int H, int N, int d);
int fa_bwd_row_tile(int d);
fa_status fa_debug_fwd_trace(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, int32_t* trace, cudaStream_t stream);
fa_status fa_debug_bwd_trace(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                             int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, int32_t* trace, cudaStream_t stream);

/*
 * Debug: one of the two launches fa_bwd makes, selected by `phase`:
 * 0 = prep (D = rowsum(dO o O) and lse in log2 units, into the workspace),
 * 1 = main (recompute P; dK, dV by key tile and dQ by query tile, all
 * accumulated in TMEM). Running phases 0 and 1 in order on one stream with the
 * same arguments is exactly fa_bwd. Used to time the main kernel on its own.
 */
fa_status fa_debug_bwd_phase(int phase, fa_dtype dtype, const void* q, const void* k, const void* v,
                             const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             void* workspace, int B, int H, int N, int d, float softmax_scale, int causal,
                             const uint8_t* block_mask, cudaStream_t stream);

/*
 * Device status: synchronises `stream`, returns the status word that kernels
 * set when a device-side wait timed out (FA_OK if none), and clears it.
 */
fa_status fa_device_status(cudaStream_t stream);

/*
 * Debug: launches one CTA that waits on a barrier nothing will complete, with
 * a time limit of `timeout_ms`; the wait gives up, records FA_ERR_TIMEOUT in
 * the status word and the CTA exits normally. Used to test the time-out path.
 */
fa_status fa_debug_timeout_probe(int timeout_ms, cudaStream_t stream);

/*
 * Debug: the real forward kernel with its TMA producer issuing no load at all
 * and every device-side wait limited to `timeout_ms` (1..5000). The MMA
 * issuer's first wait (for Q) runs out, records FA_ERR_TIMEOUT in the status
 * word and raises the CTA's abort flag; every role then leaves its loop, and,
 * as nothing was issued, nothing is in flight when the CTAs exit. o and lse
 * are not written. Used to test the abort path of the production kernel
 * without a fault. Arguments otherwise as fa_fwd.
 */
fa_status fa_debug_fwd_withhold(fa_dtype dtype, const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int H, int N, int d, float softmax_scale, int causal, int timeout_ms,
                                cudaStream_t stream);

/*
 * Debug: fa_bwd with the main kernel's TMA producers issuing no load and every
 * device-side wait limited to `timeout_ms` (1..5000): the MMA issuers' first
 * waits run out (key-stationary CTAs: K/V; query-stationary CTAs: their first
 * K), record FA_ERR_TIMEOUT and raise the CTA's abort flag; every role leaves
 * its loop, the issuers wait for what they issued, and the CTAs exit. The prep
 * launch runs normally. dq, dk, dv are not written. Arguments otherwise as
 * fa_bwd.
 */
fa_status fa_debug_bwd_withhold(fa_dtype dtype, const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv, void* workspace,
                                int B, int H, int N, int d, float softmax_scale, int causal, int timeout_ms,
                                cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
