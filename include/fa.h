/*
 * fa.h: C ABI of the exact tiled attention library (libfa.so), sm_100a.
 *
 * The library computes exact scaled dot-product attention
 *     O = softmax(scale * Q K^T) V
 * tile by tile with the online-softmax recurrence (a running row max m and
 * normaliser l; the partial output is rescaled by exp(m_old - m_new) each
 * time the max grows), writing only O and the log-sum-exp L = m + ln(l).
 * The backward pass recomputes S and P from L and dO, so no N x N matrix is
 * ever written to device memory. Sources: "FlashAttention/zh", sections
 * "why standard attention is slow" (the definition), "online softmax trick",
 * "FlashAttention algorithm" (the tiled forward and L), and "backward pass
 * and recomputation"; the varlen interface (cu_seqlens, max_s, fp16/bf16
 * only, no attention-weights output) follows the FlashAttention wrapper on
 * "InternViT-6B-448px-V1-2 ... FlashAttention v1/v2" (its three execution
 * paths).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Memory.   Every pointer is a DEVICE pointer owned by the caller. The
 *           library allocates no device memory per call; its only state is
 *           a device error word. Tensors are contiguous, row-major.
 * Layouts.  Fixed length uses BSHD: q, o, dO [B, Nq, Hq, d]; k, v
 *           [B, Nk, Hkv, d]. lse is float32 [B, Hq, Nq], natural log, of the
 *           SCALED scores: lse[b,h,i] = log sum_j exp(scale * q_i . k_j).
 * Heads.    Grouped KV heads: query head h reads KV head h / (Hq / Hkv).
 * Causal.   causal = 1 masks key j for query i when j > i + (Nk - Nq)
 *           (bottom-right alignment; the pages name the causal mask but not
 *           its alignment). A query row that sees no key gets O = 0 and
 *           lse = -inf.
 * Types.    dtype selects bf16 or fp16 for q, k, v, o, dO, dq, dk, dv;
 *           accumulation is fp32; P is rounded to dtype before P V.
 * Sizes.    d must be 64 or 128. B, Hq, Hkv >= 1; Nq, Nk >= 0 (0 gives no
 *           work); Hq % Hkv == 0.
 * Alignment Every tensor pointer must be 16-byte aligned.
 * Streams.  Work is enqueued on `stream` (may be 0 = legacy default stream)
 *           and runs asynchronously; nothing is written to host memory and
 *           no call synchronises, except fa_get_last_device_error.
 * Errors.   Invalid arguments are reported before anything is launched and
 *           nothing is launched then. Launch failures give FA_ERR_CUDA.
 *           Every wait inside a kernel is bounded; a wait that runs out sets
 *           the device error word and the kernel returns early, which the
 *           host sees through fa_get_last_device_error (FA_ERR_TIMEOUT).
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fa_stream_t; /* same type as cudaStream_t */

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* null pointer, bad size, Hq % Hkv != 0, bad scale */
    FA_ERR_UNSUPPORTED = 2, /* head dim other than 64 / 128, unknown dtype, too large */
    FA_ERR_MISALIGNED = 3,  /* a tensor pointer or stride not 16-byte aligned */
    FA_ERR_CUDA = 4,        /* a CUDA runtime or driver call failed */
    FA_ERR_TIMEOUT = 5      /* a bounded device-side wait ran out (see fa_get_last_device_error) */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

/*
 * Forward, fixed length ("FlashAttention/zh", section "FlashAttention
 * algorithm": tiled online softmax, O_i / l_i and L_i = m_i + log l_i).
 *   q [B,Nq,Hq,d], k and v [B,Nk,Hkv,d]  (inputs, dtype)
 *   o [B,Nq,Hq,d] (output, dtype), lse [B,Hq,Nq] (output, float32)
 *   scale: multiplies Q K^T; pass 1/sqrt(d) for the standard definition.
 *          Must be finite and > 0.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Forward, packed variable length (the cu_seqlens / max_s varlen path of
 * the InternViT FlashAttention wrapper; key padding is handled by unpadding
 * K/V and passing their own cu_seqlens_k).
 *   q, o [total_q, Hq, d]; k, v [total_k, Hkv, d] (dtype)
 *   cu_seqlens_q, cu_seqlens_k: DEVICE int32 [num_seqs + 1], cu[0] = 0,
 *       non-decreasing; sequence s owns query rows cu_q[s] .. cu_q[s+1]-1
 *       and key rows cu_k[s] .. cu_k[s+1]-1. Lengths may be 0.
 *   total_q, total_k: the number of rows of the q/o and k/v buffers (the
 *       host-side extents of the packed tensors; cu_seqlens live on the
 *       device, so the library cannot read them without a synchronisation).
 *       No row at or past total_q is written and no row at or past total_k
 *       is read, whatever cu_seqlens hold.
 *   max_seqlen_q, max_seqlen_k: upper bounds of the lengths (grid sizing).
 *       A sequence longer than its bound (or with a negative length) is
 *       processed only up to the bound, and the kernel records it in the
 *       device error word: the next fa_get_last_device_error returns
 *       FA_ERR_INVALID_ARG. The bounds cannot be checked before the launch,
 *       because cu_seqlens are read on the device only.
 *   lse [Hq, total_q] float32.
 *   Causal alignment is bottom-right within each sequence.
 */
fa_status fa_varlen_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                        int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream);

/*
 * Sliding-window (local) attention, forward and backward: key j is visible to
 * query i iff a - window_left <= j <= a + window_right, where a = i + Nk - Nq
 * is i's bottom-right-aligned key; a negative side is unbounded. (-1, 0) is
 * the causal mask, (-1, -1) no mask. Whole key tiles outside every row's
 * window are skipped (the block-skipping of local attention, "YOLOv12 ...",
 * section 4.2, and the tile skipping of "FlashAttention/zh"); the tiles on a
 * window's edges are masked per element. A row whose window holds no key has
 * O = 0 and L = -inf.
 * Every other argument, result and error is that of fa_fwd / fa_bwd (the
 * backward takes the lse of fa_fwd_window with the same window).
 */
fa_status fa_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d,
                        float scale, int window_left, int window_right, fa_dtype dtype, fa_stream_t stream);
fa_status fa_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        int B, int Hq, int Hkv, int Nq, int Nk, int d,
                        float scale, int window_left, int window_right, fa_dtype dtype, fa_stream_t stream);

/*
 * Sliding window plus global anchor keys (the block-sparse local attention with
 * globally visible keys of "YOLOv12 ...", section 4.2: key blocks outside the window
 * are skipped, the anchor blocks are loaded for every query): key j is visible to
 * query i iff j <= a + window_right (when window_right >= 0) and
 * (j >= a - window_left or j < n_anchor), with a = i + Nk - Nq. Whole key tiles
 * that are neither anchors nor inside some row's window are skipped. n_anchor >= 0
 * (FA_ERR_INVALID_ARG otherwise); n_anchor = 0, or window_left < 0, is exactly
 * fa_fwd_window / fa_bwd_window. Fixed length. Every other argument, result and
 * error is that of fa_fwd_window / fa_bwd_window.
 */
fa_status fa_fwd_window_anchor(const void* q, const void* k, const void* v, void* o, float* lse,
                               int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                               int window_left, int window_right, int n_anchor,
                               fa_dtype dtype, fa_stream_t stream);
fa_status fa_bwd_window_anchor(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, void* workspace,
                               int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale,
                               int window_left, int window_right, int n_anchor,
                               fa_dtype dtype, fa_stream_t stream);

/*
 * Sliding-window attention on packed variable-length batches: the window of
 * fa_fwd_window / fa_bwd_window applied within every sequence (a = i + Nk_s - Nq_s
 * with that sequence's own lengths), over the packed layout and cu_seqlens of
 * fa_varlen_fwd / fa_varlen_bwd. Every other argument, result and error is that of
 * fa_varlen_fwd / fa_varlen_bwd (the backward takes the lse of
 * fa_varlen_fwd_window with the same window).
 */
fa_status fa_varlen_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                               int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                               int Hq, int Hkv, int d, float scale, int window_left, int window_right,
                               fa_dtype dtype, fa_stream_t stream);
fa_status fa_varlen_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                               const void* dout, void* dq, void* dk, void* dv, void* workspace,
                               const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                               int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                               int Hq, int Hkv, int d, float scale, int window_left, int window_right,
                               fa_dtype dtype, fa_stream_t stream);

/*
 * The window with global anchor keys (fa_fwd_window_anchor / fa_bwd_window_anchor) on
 * packed variable-length batches: within every sequence its first n_anchor keys are
 * the anchors (key j of sequence s, counted from cu_seqlens_k[s], is visible to its
 * query i iff j <= a + window_right (when window_right >= 0) and (j >= a - window_left
 * or j < n_anchor), a = i + Nk_s - Nq_s). n_anchor >= 0 (FA_ERR_INVALID_ARG
 * otherwise); n_anchor = 0, or window_left < 0, is exactly fa_varlen_fwd_window /
 * fa_varlen_bwd_window. Every other argument, result and error is that of those calls.
 */
fa_status fa_varlen_fwd_window_anchor(const void* q, const void* k, const void* v, void* o, float* lse,
                                      const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                                      int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                                      int Hq, int Hkv, int d, float scale, int window_left, int window_right,
                                      int n_anchor, fa_dtype dtype, fa_stream_t stream);
fa_status fa_varlen_bwd_window_anchor(const void* q, const void* k, const void* v, const void* o,
                                      const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                      void* workspace, const int* cu_seqlens_q, const int* cu_seqlens_k,
                                      int num_seqs, int total_q, int total_k, int max_seqlen_q,
                                      int max_seqlen_k, int Hq, int Hkv, int d, float scale,
                                      int window_left, int window_right, int n_anchor,
                                      fa_dtype dtype, fa_stream_t stream);

/*
 * Key-padding masks of any shape (not only a tail of each sequence): key j of
 * batch b takes part iff bit j % 32 of key_bits[b * ceil(Nk/32) + j / 32] is set,
 * on top of the causal mask when causal = 1; a query row left with no key gets
 * O = 0 and lse = -inf. This is the general boolean key mask the unpad -> varlen
 * path of the InternViT FlashAttention wrapper can only express as a tail; key
 * tiles with every bit set pay nothing for it.
 *   key_bits: DEVICE uint32 [B, ceil(Nk/32)], 4-byte aligned (bits past Nk ignored).
 *   fa_pack_key_mask builds it from a DEVICE byte mask keep [B, Nk] (non-zero =
 *   keep), asynchronously on `stream`.
 * Every other argument, result and error is that of fa_fwd / fa_bwd (the backward
 * takes the lse of fa_fwd_keymask with the same mask).
 */
fa_status fa_pack_key_mask(const unsigned char* keep, unsigned int* key_bits, int B, int Nk, fa_stream_t stream);
fa_status fa_fwd_keymask(const void* q, const void* k, const void* v, void* o, float* lse,
                         const unsigned int* key_bits, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal, fa_dtype dtype, fa_stream_t stream);
fa_status fa_bwd_keymask(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace,
                         const unsigned int* key_bits, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Forward with the query/key RMS normalisation fused in front of attention
 * (the InternViT attention applies an RMSNorm to Q and K, per head, just
 * before its FlashAttention call): with
 *     q_hat = q / sqrt(mean_c(q_c^2) + eps),  k_hat = k / sqrt(mean_c(k_c^2) + eps)
 * per (token, head) row over the d values (unit gain), computed in fp32 and
 * rounded to dtype, the result is fa_fwd(q_hat, k_hat, v). q is read raw and
 * normalised in shared memory inside the attention kernel (no extra pass over
 * HBM); k is normalised once, by a row kernel, into `workspace` (each K tile
 * serves many query tiles, so normalising it there would repeat the work).
 *   workspace: device buffer of fa_fwd_qk_rmsnorm_workspace_size(B,Nk,Hkv,d)
 *       bytes, 16-byte aligned, owned by the caller; on exit it holds k_hat.
 *   eps must be finite and >= 0 (FA_ERR_INVALID_ARG). Fixed length only.
 * Every other argument, result and error is that of fa_fwd.
 */
size_t fa_fwd_qk_rmsnorm_workspace_size(int B, int Nk, int Hkv, int d);
fa_status fa_fwd_qk_rmsnorm(const void* q, const void* k, const void* v, void* o, float* lse, void* workspace,
                            int B, int Hq, int Hkv, int Nq, int Nk, int d,
                            float scale, int causal, float eps, fa_dtype dtype, fa_stream_t stream);

/*
 * Forward on strided views: the same computation as fa_fwd / fa_varlen_fwd
 * for q, k, v, o that are not contiguous, e.g. the packed QKV layout
 * (B, S, 3, H, d) of the InternViT FlashAttention wrapper, where q, k and v
 * are views into one buffer (q_strides = {S*3*H*d, 3*H*d, d}, k at +H*d,
 * v at +2*H*d), or a (B, H, S, d) layout.
 *   *_strides: HOST arrays of element strides, read before the call returns.
 *       fa_fwd_strided: {batch, token, head}; fa_varlen_fwd_strided: {token,
 *       head} (the packed buffers have no batch dimension). Every stride must
 *       be > 0 (FA_ERR_INVALID_ARG) and a multiple of 8 elements, 16 bytes
 *       (FA_ERR_MISALIGNED); the last dimension d is contiguous. o must not
 *       overlap itself or the inputs.
 *   lse keeps the contiguous layouts of fa_fwd / fa_varlen_fwd.
 * Every other argument, result and error is that of fa_fwd / fa_varlen_fwd.
 */
fa_status fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                         const long long* q_strides, const long long* k_strides,
                         const long long* v_strides, const long long* o_strides,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal, fa_dtype dtype, fa_stream_t stream);

fa_status fa_varlen_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse,
                                const long long* q_strides, const long long* k_strides,
                                const long long* v_strides, const long long* o_strides,
                                const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                                int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                                int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                                fa_stream_t stream);

/*
 * FP8 forward: the forward of fa_fwd on E4M3 inputs with per-block scaling
 * ("FlashAttention/zh", section "variants": FlashAttention-3's FP8 support; the
 * algorithm is that of fa_fwd). The real inputs are
 *     Q[b, i, h, :] = q_scale[b, h, i / 128] * e4m3(q[b, i, h, :])
 * and likewise K, V with k_scale, v_scale [b, kv head, j / 128]: one float32
 * dequantisation factor per 128 tokens of one head. Both products run on the
 * tensor core's 8-bit path; the probabilities P are rounded to E4M3 before the
 * P V product (times v_j / v_max, the block's share of the largest V factor the
 * query tile meets, which keeps them in E4M3's range), so O carries that rounding
 * (relative 2^-4 per weight, or 2^-10 absolute below E4M3's normal range); O is
 * normalised by the exact sum of P, and lse is that of the exact scores.
 *   q [B,Nq,Hq,d], k and v [B,Nk,Hkv,d]: E4M3 bytes (1 sign, 4 exponent bits
 *       with bias 7, 3 mantissa bits; 0x7F / 0xFF are NaN), 16-byte aligned.
 *   q_scale [B,Hq,ceil(Nq/128)], k_scale and v_scale [B,Hkv,ceil(Nk/128)]:
 *       DEVICE float32, finite and > 0 (not checked: they live on the device).
 *   o [B,Nq,Hq,d] bf16, lse [B,Hq,Nq] float32, as fa_fwd.
 *   d must be 128 (FA_ERR_UNSUPPORTED). Every other argument, result and error is
 *   that of fa_fwd.
 */
fa_status fa_fwd_fp8(const void* q, const void* k, const void* v,
                     const float* q_scale, const float* k_scale, const float* v_scale,
                     void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d,
                     float scale, int causal, fa_stream_t stream);

/*
 * Size in bytes of the caller-owned workspace fa_bwd needs: the per-row
 * D_i = sum_c dO_ic O_ic (float32 [B,Hq,Nq]) and the float32 dQ accumulator
 * (B*Hq*Nq*64 floats for d = 64; B*Hq*ceil(Nq/4)*4*128 floats for d = 128,
 * whose layout groups four queries), each rounded up to 256 bytes. Returns 0
 * for invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int Hq, int Nq, int d);

/*
 * Backward, fixed length ("FlashAttention/zh", section "backward pass and
 * recomputation": S and P are recomputed from the saved L and dO). With
 * P = exp(scale Q K^T - L) the gradients are the exact derivatives of the
 * definition: dV = P^T dO, dP = dO V^T, D_i = sum_c dO_ic O_ic,
 * dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q; with grouped KV
 * heads dK and dV of a KV head sum over its query heads.
 *   q, k, v, o, lse: exactly as given to / returned by fa_fwd.
 *   dout [B,Nq,Hq,d] (input, dtype).
 *   dq [B,Nq,Hq,d], dk and dv [B,Nk,Hkv,d] (outputs, dtype; overwritten).
 *   workspace: device buffer of fa_bwd_workspace_size(B,Hq,Nq,d) bytes,
 *       16-byte aligned, owned by the caller; its contents on entry do not
 *       matter and on exit are unspecified.
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dout, void* dq, void* dk, void* dv, void* workspace,
                 int B, int Hq, int Hkv, int Nq, int Nk, int d,
                 float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Backward on strided views: the gradients of fa_fwd / fa_fwd_strided for q, k, v,
 * o, dout, dq, dk, dv that are not contiguous, e.g. the packed QKV layout
 * (B, S, 3, H, d) with its gradient dqkv in the same layout (dq, dk, dv views at
 * +0, +H*d, +2*H*d of one buffer). *_strides: HOST arrays {batch, token, head}
 * of element strides with the rules of fa_fwd_strided; dq, dk and dv must not
 * overlap each other or the inputs. lse and the workspace keep their layouts.
 * Every other argument, result and error is that of fa_bwd.
 */
fa_status fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv, void* workspace,
                         const long long* q_strides, const long long* k_strides, const long long* v_strides,
                         const long long* o_strides, const long long* do_strides, const long long* dq_strides,
                         const long long* dk_strides, const long long* dv_strides,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Size in bytes of the caller-owned workspace fa_varlen_bwd needs: D
 * (float32 [Hq,total_q]) and the float32 dQ accumulator
 * (num_seqs*Hq*max_seqlen_q*64 floats for d = 64,
 * num_seqs*Hq*ceil(max_seqlen_q/4)*4*128 floats for d = 128: each sequence padded
 * to max_seqlen_q), each rounded up to 256 bytes. d must be 64 or 128; returns 0
 * for invalid sizes.
 */
size_t fa_varlen_bwd_workspace_size(int num_seqs, int total_q, int max_seqlen_q, int Hq, int d);

/*
 * Backward, packed variable length: the gradients of fa_varlen_fwd, with
 * the mathematics of fa_bwd applied to every sequence on its own ("FlashAttention/zh",
 * section "backward pass and recomputation"; the varlen layout of the
 * InternViT FlashAttention wrapper).
 *   q, k, v, o, lse, cu_seqlens_q/k, num_seqs, total_q/k, max_seqlen_q/k:
 *       exactly as given to / returned by fa_varlen_fwd.
 *   dout [total_q, Hq, d] (input, dtype).
 *   dq [total_q, Hq, d], dk and dv [total_k, Hkv, d] (outputs, dtype): rows
 *       that belong to a sequence are overwritten; rows outside every
 *       sequence are left as they were.
 *   workspace: device buffer of fa_varlen_bwd_workspace_size(...) bytes,
 *       16-byte aligned, owned by the caller.
 *   d is 64 or 128, as for fa_varlen_fwd. Causal alignment is bottom-right
 *   within each sequence.
 */
fa_status fa_varlen_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace,
                        const int* cu_seqlens_q, const int* cu_seqlens_k, int num_seqs,
                        int total_q, int total_k, int max_seqlen_q, int max_seqlen_k,
                        int Hq, int Hkv, int d, float scale, int causal, fa_dtype dtype,
                        fa_stream_t stream);

/*
 * Backward of packed variable-length batches on strided views: the gradients of
 * fa_varlen_fwd / fa_varlen_fwd_strided for q, k, v, o, dout, dq, dk, dv that are not
 * contiguous, e.g. a packed (total, 3, H, d) QKV buffer with its gradient dqkv in the
 * same layout. *_strides: HOST arrays {token, head} of element strides with the rules
 * of fa_varlen_fwd_strided; dq, dk and dv must not overlap each other or the inputs.
 * lse and the workspace keep their layouts. Every other argument, result and error is
 * that of fa_varlen_bwd.
 */
fa_status fa_varlen_bwd_strided(const void* q, const void* k, const void* v, const void* o,
                                const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                void* workspace, const long long* q_strides,
                                const long long* k_strides, const long long* v_strides,
                                const long long* o_strides, const long long* do_strides,
                                const long long* dq_strides, const long long* dk_strides,
                                const long long* dv_strides, const int* cu_seqlens_q,
                                const int* cu_seqlens_k, int num_seqs, int total_q, int total_k,
                                int max_seqlen_q, int max_seqlen_k, int Hq, int Hkv, int d,
                                float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Decode: attention of the Nq newest query tokens of each sequence against a
 * long key/value cache (Nq = 1 for one generated token, a few for speculative
 * decoding), by the same tiled online softmax as the forward ("FlashAttention/zh",
 * section "FlashAttention algorithm"), with the keys split across the GPU:
 * the key tiles of all (sequence, KV head) pairs are laid end to end and every
 * CTA takes an equal share; each share leaves a partial output and its
 * log-sum-exp, and a second kernel merges the shares of each pair with
 * L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s (the online-softmax
 * rescale applied to whole partial results; exact up to rounding). The query
 * heads that share a KV head are one tile, so each K/V row is read from HBM
 * once. The paged cache is the block-tiled KV cache of PagedAttention (named
 * on "FlashAttention/zh", section "variants").
 *   q [B,Nq,Hq,d] (dtype); o [B,Nq,Hq,d] (dtype), lse [B,Hq,Nq] (float32):
 *       the layouts of fa_fwd.
 *   fa_decode: k, v [B,Nk,Hkv,d], the caches (Nk = their capacity).
 *   fa_decode_paged: k_pages, v_pages [num_pages,page_size,Hkv,d] page pools;
 *       block_table DEVICE int32 [B,max_pages]: key position p of sequence b is
 *       row p % page_size of page block_table[b*max_pages + p/page_size]. Entries
 *       for positions past the sequence's length are not read; a page index
 *       outside [0, num_pages) reads zeros. page_size must be 16, 32 or a
 *       multiple of 64 (FA_ERR_UNSUPPORTED otherwise).
 *   cache_seqlens: DEVICE int32 [B] or NULL (fa_decode only): sequence b uses
 *       keys 0 .. cache_seqlens[b]-1, clamped to [0, capacity] (capacity = Nk,
 *       or max_pages*page_size); NULL = every sequence uses all Nk keys. Rows
 *       of the cache past a sequence's length may hold anything, NaN included.
 *       Required (non-NULL) for fa_decode_paged.
 *   causal: query token t of a sequence with n keys sees keys 0 .. t + n - Nq
 *       (bottom-right alignment, as fa_fwd). A row that sees no key (n = 0, or
 *       t + n - Nq < 0) gets O = 0 and lse = -inf.
 *   workspace: device buffer of fa_decode_workspace_size(B,Hq,Hkv,Nq,d) bytes,
 *       16-byte aligned, owned by the caller, for the partial results. The size
 *       depends on the SM count of the CURRENT device: query it with the device
 *       the call will run on current (0 when no device is visible).
 *   (Hq / Hkv) * Nq must be at most 128 (FA_ERR_UNSUPPORTED otherwise; use
 *   fa_fwd for longer query blocks). Every other argument, result and error
 *   is that of fa_fwd; cache_seqlens and block_table must be 4-byte aligned.
 */
size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Nq, int d);
fa_status fa_decode(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int* cache_seqlens, void* workspace,
                    int B, int Hq, int Hkv, int Nq, int Nk, int d,
                    float scale, int causal, fa_dtype dtype, fa_stream_t stream);
fa_status fa_decode_paged(const void* q, const void* k_pages, const void* v_pages, void* o, float* lse,
                          const int* cache_seqlens, const int* block_table, void* workspace,
                          int B, int Hq, int Hkv, int Nq, int num_pages, int page_size, int max_pages, int d,
                          float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Backward without a caller-provided workspace. This entry point has no
 * counterpart in the pages; it exists for callers that cannot allocate
 * device memory themselves (a host framework that owns every allocation,
 * a loop that must not pay for cudaMalloc's device-wide synchronisation, a
 * plugin with a fixed memory budget).
 *
 * Same arguments, results and errors as fa_bwd, minus `workspace`: the
 * workspace is a device array of FA_BWD_NOALLOC_MAX_BYTES bytes inside the
 * library, which every GPU that loads this part of the library keeps until
 * the process exits. Under CUDA's lazy module loading (the default,
 * CUDA_MODULE_LOADING=LAZY) a GPU loads it when fa_bwd_noalloc first runs
 * there; under CUDA_MODULE_LOADING=EAGER every GPU context the process
 * creates loads it, and holds the 64 MiB, whether or not fa_bwd_noalloc is
 * ever called. Nothing is allocated per call: no cudaMalloc, no cudaFree,
 * no allocating library routine.
 *   - Sizes whose fa_bwd_workspace_size(B, Hq, Nq, d) exceeds
 *     FA_BWD_NOALLOC_MAX_BYTES are rejected with FA_ERR_UNSUPPORTED before
 *     anything runs (with d = 128: B * Hq * Nq up to about 130,000 rows).
 *   - The first call on a device looks up the array's device address (a
 *     one-time set-up per device, done with that device current); make that
 *     first call before any stream capture.
 *   - All calls share the one array: calls whose work overlaps on the GPU
 *     (different streams, or different host threads, without ordering
 *     between them) race on it and give wrong gradients. Calls ordered on
 *     one stream are safe; each call re-initialises what it reads.
 */
#define FA_BWD_NOALLOC_MAX_BYTES (64u << 20)

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dout, void* dq, void* dk, void* dv,
                         int B, int Hq, int Hkv, int Nq, int Nk, int d,
                         float scale, int causal, fa_dtype dtype, fa_stream_t stream);

/*
 * Profiling aid: when `before` and `after` are both non-NULL CUDA event
 * handles (cudaEvent_t), every later fa_bwd call records `before` on its
 * stream right before it launches its main kernel and `after` right after,
 * so a caller can time that kernel alone with cudaEventElapsedTime. Passing
 * NULL turns it off. The setting is process-wide and not synchronised
 * between host threads; the events must stay valid while it is set.
 */
void fa_bwd_set_timing_events(void* before, void* after);

/* A static description of a status code. Never NULL. */
const char* fa_status_string(fa_status s);

/*
 * Synchronises `stream`, then reports and clears the current device's error
 * word (each GPU has its own; a kernel records into the word of the device it
 * runs on): FA_ERR_TIMEOUT if a kernel gave up on a bounded wait since the
 * last call, FA_ERR_INVALID_ARG if a varlen kernel met a sequence longer than
 * its max_seqlen bound, FA_ERR_CUDA if the synchronisation failed or a kernel
 * refused to run, FA_OK otherwise.
 */
fa_status fa_get_last_device_error(fa_stream_t stream);

/* The raw device error code behind the last non-OK fa_get_last_device_error:
 * 0x1000 + site for a wait that ran out, 0x2000 for a shared-memory window
 * that was not 1024-byte aligned (the kernel then does nothing); 0 if none. */
int fa_get_last_device_error_site(void);

/*
 * Self-test of the failure path (no counterpart in the pages): launches one
 * CTA that waits, with the same bounded wait every kernel uses, on a barrier
 * that nothing arrives on. About 2 s later the wait gives up and records its
 * site (0x1000 + 99) in the device error word, and the kernel returns; the
 * caller sees FA_ERR_TIMEOUT from fa_get_last_device_error and the context
 * stays usable. Returns the launch status.
 */
fa_status fa_selftest_bounded_wait(fa_stream_t stream);

/* Library version, "major.minor.patch". */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
