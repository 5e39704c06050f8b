/*
 * fa.h -- C ABI of the B200 (sm_100a) exact-attention library.
 *
 * Exact scaled-dot-product attention
 *     O = softmax(S) V,   S = scale * Q K^T  (+ score modifiers, + mask),
 * computed tile by tile with an online softmax so that neither the score
 * matrix S nor the probability matrix P ever reaches device memory, plus the
 * per-row natural log-sum-exp LSE_i = ln sum_j exp(S_ij): the forward (fixed
 * length, packed sequences, packed QKV, grouped-query heads), the paged
 * split-KV decode (with the cache append), and the backward (dQ, dK, dV).
 *
 * Sources (web pages about FlashAttention; their formulas were lost in
 * extraction, so the readings below state the plain form that the rest of the
 * text supports):
 *   - standard attention and its N x N intermediates: "FlashAttention及变种改进",
 *     section 二.1 "标准自注意力的计算瓶颈";
 *   - tiling into on-chip blocks, online (row-block) softmax, async copy
 *     overlapped with compute: "IO感知技术革命：FlashAttention如何重塑大模型训练的
 *     经济学", sections "分块计算的投资回报模型", "在线Softmax的现金流优化",
 *     "异步执行的供应链思维"; softmax fused with both matmuls:
 *     "FlashAttention深度解析", section "重新定义注意力计算";
 *   - bottom-right causal alignment, split-KV decode with a merge kernel,
 *     sliding window, ALiBi, paged KV cache through a block table, tanh
 *     softcapping: "Flash-Attention v2.0 到 v2.7 更新", opening paragraph and
 *     sections v2.1, v2.2, v2.3, v2.4, v2.5, v2.6.
 *
 * Conventions shared by the calls
 *   - Every tensor pointer is a DEVICE pointer to contiguous memory, 16-byte
 *     aligned, owned by the caller. The library allocates nothing, keeps no
 *     pointer after a call returns and holds no global state besides a
 *     per-device cache of device properties and the fixed device array of
 *     fa_fwd_kvcache_noalloc.
 *   - Element types: Q, K, V and O are fp16 or bf16 (fa_dtype), or for
 *     fa_fwd_fp8 8-bit Q, K, V (fa_fp8_format) and bf16 O; LSE is fp32;
 *     block tables and lengths are int32; ALiBi slopes are fp32. Arithmetic
 *     is fp32 (the two products run on tensor cores with fp32 accumulation).
 *   - Score modifiers, applied in this order to s = scale * (q . k):
 *       softcap > 0:   s = softcap * tanh(s / softcap)
 *       alibi_slopes:  s += -alibi_slopes[h] * |pos_i - j|
 *       mask:          s = -inf for every key j that query i may not see.
 *     Query row i (0-based) of Nq sits at key position pos_i = i + Nk - Nq
 *     (bottom-right alignment: the last query meets the last key). Key j is
 *     visible iff
 *       (!causal || j <= pos_i) and
 *       (window_left  < 0 || j >= pos_i - window_left) and
 *       (window_right < 0 || j <= pos_i + window_right).
 *   - A query row that sees no key gets O = 0 and LSE = -inf.
 *   - Calls are asynchronous on `stream` (0 = legacy default stream): they
 *     validate their arguments, enqueue kernels and return; they never
 *     synchronise. Invalid arguments are reported before anything is
 *     enqueued; FA_ERR_CUDA reports a failed launch or CUDA call.
 *   - Requires a compute-capability 10.0 device (B200); elsewhere the calls
 *     return FA_ERR_DEVICE.
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_NULL = 1,      /* a required pointer is NULL */
    FA_ERR_SHAPE = 2,     /* a size is negative or beyond a stated limit */
    FA_ERR_DTYPE = 3,     /* dtype is not FA_FP16 / FA_BF16 */
    FA_ERR_HEADDIM = 4,   /* d is not 64 or 128 */
    FA_ERR_ARG = 5,       /* scale/softcap not finite or negative cap, window < -1,
                             page_size < 1, num_splits outside [0, FA_MAX_SPLITS],
                             or a pointer not 16-byte aligned */
    FA_ERR_WORKSPACE = 6, /* split-KV workspace missing, misaligned or too small */
    FA_ERR_CUDA = 7,      /* a CUDA runtime/driver call or a launch failed */
    FA_ERR_DEVICE = 8     /* no device, or the current device is not sm_100 */
} fa_status;

typedef enum { FA_FP16 = 0, FA_BF16 = 1 } fa_dtype;
typedef enum { FA_E4M3 = 0, FA_E5M2 = 1 } fa_fp8_format;

#define FA_MAX_SPLITS 64

/*
 * fa_fwd -- tiled attention forward (prefill / training shape).
 *
 *   q    [B, Nq, H, d]   fp16/bf16, read
 *   k, v [B, Nk, H, d]   fp16/bf16, read
 *   out  [B, Nq, H, d]   same dtype, written
 *   lse  [B, H, Nq]      fp32, written (natural log)
 *   scale                multiplies q . k (typically 1/sqrt(d)); finite
 *   causal               0/1, bottom-right aligned as above
 *   window_left/right    -1 = unbounded, else >= 0 (inclusive bounds)
 *   alibi_slopes         [H] fp32 device array, or NULL for no ALiBi
 *   softcap              0 = off, else > 0 and finite
 *
 * Limits: B, H, Nq, Nk >= 0; B*H < 2^31; Nq, Nk <= 2^28. B*H*Nq == 0 is a
 * no-op; Nk == 0 makes every row empty. d is 64 or 128. out must not alias
 * q, k or v.
 */
fa_status fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse,
                 int B, int H, int Nq, int Nk, int d, fa_dtype dtype, float scale,
                 int causal, int window_left, int window_right,
                 const float *alibi_slopes, float softcap, cudaStream_t stream);

/*
 * fa_fwd_fp8 -- the forward on 8-bit inputs. "FlashAttention深度解析：从算法
 * 创新到产业变革的全面影响" (section 未来展望) and "IO感知技术革命" (section
 * H100架构的性能跃升) name an FP8 forward without stating its form; the
 * reading taken: q, k, v hold 8-bit floats x8 that stand for x8 * descale_x
 * (one fp32 factor per tensor), and the result is fa_fwd's attention of
 * those dequantised values, written as bf16.
 *
 *   q    [B, Nq, H, d]      8-bit (fmt), read
 *   k, v [B, Nk, H_kv, d]   8-bit (fmt), read (H % H_kv == 0, as fa_fwd_gqa)
 *   out  [B, Nq, H, d]      bf16, written
 *   lse  [B, H, Nq]         fp32, written (natural log)
 *   fmt                     FA_E4M3 or FA_E5M2 (all three tensors), else
 *                           FA_ERR_DTYPE
 *   scale, descale_q/k/v    the scores are (scale * descale_q * descale_k) *
 *                           (q8 . k8), O is scaled by descale_v; the
 *                           descales finite and > 0, else FA_ERR_ARG
 *   causal, windows, alibi_slopes, softcap   as in fa_fwd
 *   workspace               device buffer of fa_fwd_fp8_workspace_size()
 *                           bytes, 16-byte aligned, caller-owned (V is
 *                           transposed into it first, so both products read
 *                           K-major 8-bit operands), else FA_ERR_WORKSPACE
 *
 * Both products run on the tensor cores with 8-bit operands (kind::f8f6f4,
 * fp32 accumulation); P is rounded to fmt before the PV product (relative
 * error 2^-4 for E4M3, 2^-3 for E5M2, larger for values below the format's
 * normal range), and O is divided by the sum of P as rounded, so those
 * roundings perturb the weights of a convex combination of V rows. d must be
 * 128 (FA_ERR_HEADDIM otherwise). Other limits as in fa_fwd.
 */
size_t fa_fwd_fp8_workspace_size(int B, int H_kv, int Nk, int d);
fa_status fa_fwd_fp8(const void *q, const void *k, const void *v, void *out, float *lse,
                     int B, int H, int H_kv, int Nq, int Nk, int d, fa_fp8_format fmt,
                     float scale, float descale_q, float descale_k, float descale_v,
                     int causal, int window_left, int window_right,
                     const float *alibi_slopes, float softcap,
                     void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_fwd_gqa -- fa_fwd with grouped-query attention: H query heads share
 * H_kv key/value heads. The pages do not define this form; the reading
 * taken is the plain one: query head h attends with K/V head h / (H / H_kv),
 * and everything else is exactly fa_fwd.
 *
 *   k, v [B, Nk, H_kv, d]  (q, out, lse as in fa_fwd)
 *   H_kv                   1 <= H_kv <= H and H % H_kv == 0, else FA_ERR_SHAPE
 *                          (H_kv == H is fa_fwd; H_kv == 1 is multi-query)
 */
fa_status fa_fwd_gqa(const void *q, const void *k, const void *v, void *out, float *lse,
                     int B, int H, int H_kv, int Nq, int Nk, int d, fa_dtype dtype, float scale,
                     int causal, int window_left, int window_right,
                     const float *alibi_slopes, float softcap, cudaStream_t stream);

/*
 * fa_fwd_qkvpacked -- fa_fwd with Q, K and V packed in one tensor, the
 * layout of the interface "FlashAttention深度解析：从算法创新到产业变革的全面
 * 影响" names beside the separate one (flash_attn_qkvpacked_func):
 *
 *   qkv  [B, N, 3, H, d]  fp16/bf16, read; qkv[b, n, 0] is q[b, n],
 *                         qkv[b, n, 1] is k[b, n], qkv[b, n, 2] is v[b, n]
 *   out  [B, N, H, d]     written;  lse [B, H, N] fp32, written
 *
 * Nq = Nk = N; every other argument, limit and error as in fa_fwd. Nothing
 * is copied: the kernel reads q, k and v in place through strided maps.
 */
fa_status fa_fwd_qkvpacked(const void *qkv, void *out, float *lse, int B, int H, int N, int d,
                           fa_dtype dtype, float scale, int causal, int window_left, int window_right,
                           const float *alibi_slopes, float softcap, cudaStream_t stream);

/*
 * fa_fwd_varlen_qkvpacked -- fa_fwd_varlen with Q, K and V packed:
 * qkv [total, 3, H, d], out [total, H, d], lse [H, total]; one offset array
 * cu_seqlens [B + 1] (device int32) for queries and keys alike, and one
 * bound max_seqlen. Every other argument as in fa_fwd_varlen.
 */
fa_status fa_fwd_varlen_qkvpacked(const void *qkv, void *out, float *lse, const int *cu_seqlens,
                                  int B, int H, int max_seqlen, int total, int d, fa_dtype dtype,
                                  float scale, int causal, int window_left, int window_right,
                                  const float *alibi_slopes, float softcap, cudaStream_t stream);

/*
 * fa_fwd_varlen -- fa_fwd over a batch of sequences of different lengths
 * packed along the token axis ("FlashAttention深度解析：从算法创新到产业变革的
 * 全面影响", section 未来展望, names variable sequence lengths among the
 * features being added). The pages give no formula for it: each sequence b
 * is attended exactly as fa_fwd would attend it alone, with its own Nq_b,
 * Nk_b and the same bottom-right causal alignment, window, ALiBi and
 * softcap rules.
 *
 *   q    [total_q, H, d]  fp16/bf16, read; sequence b owns rows
 *                         cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k, v [total_k, H, d]  fp16/bf16, read; rows cu_seqlens_k[b] ..
 *   out  [total_q, H, d]  same dtype, written (rows of the sequences only)
 *   lse  [H, total_q]     fp32, written (natural log)
 *   cu_seqlens_q, cu_seqlens_k
 *                         [B + 1] int32 DEVICE arrays of row offsets:
 *                         nondecreasing, [0] = 0, [B] <= total, and every
 *                         length at most max_seqlen_q / max_seqlen_k
 *   max_seqlen_q, max_seqlen_k  bounds of the lengths (the grid is sized
 *                         from max_seqlen_q)
 *   the remaining arguments as in fa_fwd
 *
 * The offsets are read on the device only (no synchronisation): a sequence
 * whose entries break the contract is skipped and its rows are left as
 * they were; no memory outside the buffers is touched. Limits: B, H >= 0,
 * total_q, total_k >= 0 and <= 2^28, B*H < 2^31. B*H*max_seqlen_q == 0 or
 * total_q == 0 is a no-op.
 */
fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *out, float *lse,
                        const int *cu_seqlens_q, const int *cu_seqlens_k,
                        int B, int H, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                        int d, fa_dtype dtype, float scale,
                        int causal, int window_left, int window_right,
                        const float *alibi_slopes, float softcap, cudaStream_t stream);

/*
 * fa_fwd_kvcache -- split-KV ("flash-decoding") attention of one new query
 * token per sequence over a paged KV cache.
 *
 *   q             [B, 1, H, d]                      fp16/bf16, read
 *   k_cache,
 *   v_cache       [num_pages, page_size, H, d]      fp16/bf16, read
 *   block_table   [B, max_blocks] int32: token t of sequence b is row
 *                 t % page_size of page block_table[b][t / page_size]
 *   cache_seqlens [B] int32: L_b, the number of cached tokens of sequence b
 *                 (the new token's own k/v must already be in the cache)
 *   out           [B, 1, H, d]                      same dtype, written
 *   lse           [B, H, 1]                         fp32, written
 *   window_left   -1 = unbounded, else keys j >= L_b - 1 - window_left
 *   alibi_slopes  [H] fp32 or NULL;  softcap as in fa_fwd
 *   num_splits    0 = automatic (fa_kvcache_num_splits), else 1..FA_MAX_SPLITS
 *   workspace     device scratch of at least fa_kvcache_workspace_size(...)
 *                 bytes, 16-byte aligned; may be NULL when that size is 0.
 *                 Its contents on entry do not matter; it is clobbered.
 *
 * The query sits at position L_b - 1, so causally it sees all L_b keys (the
 * decode example of bottom-right alignment). Each sequence's visible keys are
 * cut into num_splits contiguous ranges of equal whole-page length; a
 * split kernel computes a partial (O_s, LSE_s) per range and, when more than
 * one split is used, a merge kernel forms LSE = ln sum_s exp(LSE_s) and
 * O = sum_s exp(LSE_s - LSE) O_s.
 *
 * Device-side values cannot be checked before launch. An L_b outside
 * [0, max_blocks * page_size] or a referenced block-table entry outside
 * [0, num_pages) is never dereferenced; that sequence's O and LSE rows are
 * set to NaN instead. L_b == 0 gives O = 0, LSE = -inf.
 *
 * Limits: B >= 0 (0 is a no-op), H >= 1, B*H*FA_MAX_SPLITS < 2^31,
 * num_pages >= 1, page_size >= 1, max_blocks >= 1,
 * max_blocks * page_size < 2^31.
 */
fa_status fa_fwd_kvcache(const void *q, const void *k_cache, const void *v_cache,
                         const int *block_table, const int *cache_seqlens,
                         void *out, float *lse,
                         int B, int H, int d, int num_pages, int page_size, int max_blocks,
                         fa_dtype dtype, float scale, int window_left,
                         const float *alibi_slopes, float softcap, int num_splits,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_fwd_kvcache_gqa -- fa_fwd_kvcache with grouped-query attention: the
 * caches hold H_kv heads ([num_pages, page_size, H_kv, d]); query head h
 * attends with cache head h / (H / H_kv). 1 <= H_kv <= H and H % H_kv == 0,
 * else FA_ERR_SHAPE. Workspace size and every other argument as for
 * fa_fwd_kvcache with the same B, H, d (fa_kvcache_num_splits and
 * fa_kvcache_workspace_size take H, the query heads). With num_splits = 0
 * and several query heads per cache head, the automatic count may be lower
 * than fa_kvcache_num_splits reports (one CTA serves a group of query heads
 * and reads its cache head once), never higher, so that workspace suffices.
 */
fa_status fa_fwd_kvcache_gqa(const void *q, const void *k_cache, const void *v_cache,
                             const int *block_table, const int *cache_seqlens,
                             void *out, float *lse,
                             int B, int H, int H_kv, int d, int num_pages, int page_size,
                             int max_blocks, fa_dtype dtype, float scale, int window_left,
                             const float *alibi_slopes, float softcap, int num_splits,
                             void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_kvcache_append -- writes n_new new tokens per sequence into the paged
 * caches: token i of sequence b (k_new[b, i], v_new[b, i]) goes to position
 * t = cache_seqlens[b] + i, i.e. row t % page_size of page
 * block_table[b][t / page_size] ("Flash-Attention v2.0 到 v2.7 更新", v2.5: the
 * paged cache; "解密FlashAttention：如何让大语言模型推理速度翻倍", section
 * 智能緩存機制: the key-value cache keeps the context already processed).
 * cache_seqlens is read, not updated: the caller advances it by n_new
 * before the next decode call.
 *
 *   k_new, v_new  [B, n_new, H_kv, d] fp16/bf16 device, read
 *   k_cache, v_cache  [num_pages, page_size, H_kv, d] same dtype, written
 *                 at the new positions only
 *   block_table [B, max_blocks], cache_seqlens [B]  int32 device, read
 *
 * Positions at or past max_blocks * page_size, negative lengths and table
 * entries outside [0, num_pages) are skipped on the device (nothing is
 * written for them). Limits: B <= 65535; B * n_new * H_kv < 2^31;
 * max_blocks * page_size < 2^31. B * n_new == 0 is a no-op. Pointers
 * 16-byte aligned (the int32 arrays 4-byte aligned).
 */
fa_status fa_kvcache_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                            const int *block_table, const int *cache_seqlens,
                            int B, int n_new, int H_kv, int d, int num_pages, int page_size,
                            int max_blocks, fa_dtype dtype, cudaStream_t stream);

/*
 * fa_bwd -- backward pass of fa_fwd / fa_fwd_gqa: the gradients dq, dk, dv
 * of L = sum(dout * O), where O and lse are what the forward returned for the
 * same q, k, v and options.
 *
 * The pages name the backward pass ("FlashAttention深度解析：从算法创新到产业
 * 变革的全面影响", section 技术演进, version 2.4; "Flash-Attention v2.0 到 v2.7
 * 更新", section v2.4) without its formulas; this is the gradient of the
 * forward's definition. With s = scale * q k^T softcapped, ALiBi-biased and
 * masked as in fa_fwd, P = exp(s - lse):
 *   dv = P^T dout;  dP = dout v^T;  D_i = sum_c dout_ic O_ic
 *   dS = P o (dP - D) (o (1 - tanh^2) under softcap);
 *   dq = scale * dS k;  dk = scale * dS^T q
 * Grouped-query k, v heads (H_kv < H) receive the sum over the query heads
 * that read them. P is rebuilt tile by tile from lse; no N x N array is
 * written. dk and dv are summed in a fixed order. With deterministic = 0, dq
 * is accumulated in fp32 in the workspace across key blocks with atomic
 * adds, so its last bits may differ from run to run; with deterministic = 1
 * (the deterministic backward named in "Flash-Attention v2.0 到 v2.7 更新",
 * section v2.4) a separate pass sums dq over the key blocks of each query
 * block in a fixed order, rebuilding S and dP there (about 1.4x the
 * products), and every output repeats bit for bit.
 *
 *   q, out, dout, dq   [B, Nq, H, d]       contiguous, dtype
 *   k, v, dk, dv       [B, Nk, H_kv, d]    contiguous, dtype
 *   lse                [B, H, Nq]          fp32 (the forward's, natural log)
 *   workspace          fa_bwd_workspace_size(B, H, Nq, d) bytes of device
 *                      memory, 16-byte aligned (fp32 dq accumulator, D, and
 *                      the job counters of the persistent kernels)
 *   scale, causal, window_left, window_right, alibi_slopes, softcap: as fa_fwd
 *   deterministic      0 or 1 (see above)
 * Outputs dq, dk, dv are overwritten (not accumulated). The caller owns every
 * buffer; the call only enqueues work on `stream`.
 *
 * Errors: as fa_fwd_gqa, plus FA_ERR_WORKSPACE when the workspace is missing,
 * misaligned or too small, and FA_ERR_SHAPE when ceil(Nk / 128) * B * H_kv
 * (the key-block jobs) or, with deterministic = 1, ceil(Nq / 128) * B * H
 * (the query-tile jobs) exceeds 2^31 - 1.
 * Nq == 0 gives zero dk, dv; Nk == 0 gives zero dq; B == 0 is a no-op.
 */
size_t fa_bwd_workspace_size(int B, int H, int Nq, int d);

fa_status fa_bwd(const void *q, const void *k, const void *v, const void *out, const float *lse,
                 const void *dout, void *dq, void *dk, void *dv, int B, int H, int H_kv, int Nq, int Nk,
                 int d, fa_dtype dtype, float scale, int causal, int window_left, int window_right,
                 const float *alibi_slopes, float softcap, int deterministic, void *workspace,
                 size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_bwd_varlen -- fa_bwd for packed sequences of different lengths, the
 * backward of fa_fwd_varlen (with H_kv key/value heads, H % H_kv == 0):
 *
 *   q, out, dout, dq   [total_q, H, d]     sequence b owns rows cu_seqlens_q[b] ..
 *   k, v, dk, dv       [total_k, H_kv, d]  sequence b owns rows cu_seqlens_k[b] ..
 *   lse                [H, total_q]        fp32, the forward's (natural log)
 *   cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k: as fa_fwd_varlen
 *   workspace          fa_bwd_workspace_size(1, H, total_q, d) bytes
 *   the remaining arguments as in fa_bwd
 *
 * Each sequence's gradients are those fa_bwd gives for it alone. The offsets
 * are read on the device only: a sequence whose entries break the contract
 * is skipped, its dk and dv rows left as they were; dq rows that belong to no
 * valid sequence are written as zero. Limits: total_q, total_k <= 2^28, and
 * the job counts of fa_bwd.
 */
fa_status fa_bwd_varlen(const void *q, const void *k, const void *v, const void *out, const float *lse,
                        const void *dout, void *dq, void *dk, void *dv, const int *cu_seqlens_q,
                        const int *cu_seqlens_k, int B, int H, int H_kv, int max_seqlen_q, int max_seqlen_k,
                        int total_q, int total_k, int d, fa_dtype dtype, float scale, int causal,
                        int window_left, int window_right, const float *alibi_slopes, float softcap,
                        int deterministic, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * fa_bwd_qkvpacked, fa_bwd_varlen_qkvpacked -- the backward of
 * fa_fwd_qkvpacked / fa_fwd_varlen_qkvpacked: gradients of q, k and v written
 * into one packed tensor laid out like qkv.
 *
 *   qkv               [B, N, 3, H, d] (fixed) or [total, 3, H, d] (packed)
 *   out, dout         [B, N, H, d] or [total, H, d], contiguous
 *   lse               [B, H, N] or [H, total], the forward's
 *   dqkv              like qkv, written: slot 0 dq, 1 dk, 2 dv
 *   cu_seqlens        [B + 1] device offsets (varlen form; q and k alike)
 *   workspace         fa_bwd_workspace_size(B, H, N, d), or (1, H, total, d)
 * Everything else as fa_bwd / fa_bwd_varlen (H_kv = H).
 */
fa_status fa_bwd_qkvpacked(const void *qkv, const void *out, const float *lse, const void *dout, void *dqkv,
                           int B, int H, int N, int d, fa_dtype dtype, float scale, int causal,
                           int window_left, int window_right, const float *alibi_slopes, float softcap,
                           int deterministic, void *workspace, size_t workspace_bytes, cudaStream_t stream);

fa_status fa_bwd_varlen_qkvpacked(const void *qkv, const void *out, const float *lse, const void *dout,
                                  void *dqkv, const int *cu_seqlens, int B, int H, int max_seqlen, int total,
                                  int d, fa_dtype dtype, float scale, int causal, int window_left,
                                  int window_right, const float *alibi_slopes, float softcap, int deterministic,
                                  void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Number of splits fa_fwd_kvcache uses for these sizes: num_splits itself
 * when it is 1..FA_MAX_SPLITS, else the automatic choice, which depends only
 * on B, H and the longest possible sequence max_blocks * page_size (host-side
 * sizes, so no device read is needed). Returns -1 for invalid sizes.
 */
int fa_kvcache_num_splits(int B, int H, int d, int max_blocks, int page_size, int num_splits);

/*
 * Number of splits fa_fwd_kvcache_gqa launches with H_kv cache heads: the
 * same as fa_kvcache_num_splits for an explicit num_splits or H_kv == H;
 * with grouped heads on 64-multiple pages and num_splits = 0 the automatic
 * count is aimed at the CTAs the grouped kernel launches (one per group of
 * query heads), never above fa_kvcache_num_splits(B, H, ...), so the
 * workspace fa_kvcache_workspace_size reports always suffices. Returns -1
 * for invalid sizes.
 */
int fa_kvcache_num_splits_gqa(int B, int H, int H_kv, int d, int max_blocks, int page_size, int num_splits);

/*
 * Bytes of workspace fa_fwd_kvcache needs for these sizes (0 when a single
 * split is used). Returns 0 for invalid sizes as well; fa_fwd_kvcache then
 * reports the invalid argument.
 */
size_t fa_kvcache_workspace_size(int B, int H, int d, int max_blocks, int page_size, int num_splits);

/* Size of the device array fa_fwd_kvcache_noalloc keeps its split partials in. */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/*
 * fa_fwd_kvcache_noalloc -- fa_fwd_kvcache for callers that cannot allocate
 * device memory. The pages have no counterpart to this call; it exists for
 * this library's users: a plain C host program or plugin without a device
 * allocator of its own, a component inside another runtime whose memory pool
 * already holds the free device memory (so its own cudaMalloc would fail),
 * or a latency-bound decode loop that must not call cudaMalloc, which can
 * synchronise the device.
 *
 * Arguments, layouts, results and errors are those of fa_fwd_kvcache minus
 * the workspace: the split partials go to a file-scope device array of
 * FA_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library, which every GPU that
 * loads the library holds until the process exits. The call allocates
 * nothing and calls no cudaMalloc or cudaFree.
 *   - Sizes whose partials need more than FA_NOALLOC_SCRATCH_BYTES
 *     (fa_kvcache_workspace_size(...) > FA_NOALLOC_SCRATCH_BYTES) are
 *     rejected with FA_ERR_WORKSPACE before anything is enqueued; pass a
 *     smaller explicit num_splits or use fa_fwd_kvcache.
 *   - The first call on a device that needs the array (more than one split)
 *     looks up the array's device address for that device, with that device
 *     current; make that first call before any stream capture. A failed
 *     lookup returns FA_ERR_CUDA and is not remembered: the next call on that
 *     device tries again.
 *   - All calls on a device share the one array and it keeps the last call's
 *     partials. Each call overwrites every partial it reads, so nothing needs
 *     clearing, but calls whose kernels overlap on the GPU (different streams
 *     without ordering) race on the array: order them on one stream.
 */
fa_status fa_fwd_kvcache_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                 const int *block_table, const int *cache_seqlens,
                                 void *out, float *lse,
                                 int B, int H, int d, int num_pages, int page_size, int max_blocks,
                                 fa_dtype dtype, float scale, int window_left,
                                 const float *alibi_slopes, float softcap, int num_splits,
                                 cudaStream_t stream);

/* Static, human-readable name of a status code. */
const char *fa_status_string(fa_status status);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
