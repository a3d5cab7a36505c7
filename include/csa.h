/*
 * csa.h -- C ABI of the B200 (sm_100a) DeepSeek-V4 hybrid-attention forward: Compressed Sparse
 * Attention (CSA) and Heavily Compressed Attention (HCA), prefill and decode.
 *
 * Sources for what each call computes:
 *   [HF-V4]   Hugging Face Transformers docs, "DeepSeek-V4", sections "Hybrid attention (§2.3)"
 *             and "Attention mask layout";
 *   [digest]  insight.ai.kr digest of the Hugging Face DeepSeek-V4 blog post (softmax-gated
 *             pooling with a learned position bias; ReLU multi-head lightning indexer; FP8 KV
 *             with BF16 RoPE dims);
 *   [atlas]   llm-atlas "DeepSeek-V4-Flash", table "config.json full fields" (head_dim 512,
 *             64 heads, 1 KV head, qk_rope_head_dim 64, index 64 x 128, index_topk 512,
 *             sliding_window 128, rope_theta 10000, compress_rope_theta 160000).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library allocates and
 *     frees nothing. Layouts are dense row-major with the shapes given. bf16 tensors are passed
 *     as void* (IEEE bfloat16 bit patterns), FP8 as uint8 E4M3 codes (OCP definition).
 *   - Base pointers must be 16-byte aligned; D, d_I and rope_dim as documented per call.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Argument checks run on the host
 *     before anything is launched; a failed check returns its status and launches nothing.
 *     Kernels run asynchronously in stream order; launch failures return CSA_ERR_CUDA.
 *   - `workspace` (device, caller-owned, size from csa_workspace_size) starts with a status word.
 *     Each call that takes a workspace zeroes it in stream order, then kernels record data errors
 *     found on the device (for example an index that is out of range or not yet visible; such a
 *     key is skipped). Read it with csa_get_device_status after the call.
 *   - Calls on the same workspace must not overlap on the GPU.
 *   - Nothing here aborts, traps or asserts on the device.
 *   - Prefill calls (1-5) take a chunk of S tokens at positions pos0 .. pos0+S-1 ([HF-V4 "Cache
 *     layers"]: the compressor and indexer state carries over between forward calls). Per-query
 *     tensors (q, qI, w, idx, o) hold the chunk's S rows; tensors of the whole history (kv, gate,
 *     kv_rot, C, kI) are indexed by absolute position or entry. A chunk's results equal rows
 *     pos0 .. pos0+S-1 of one prefill over positions 0 .. pos0+S-1. pos0 = 0 is a whole prefill.
 */
#ifndef CSA_B200_H
#define CSA_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define CSA_API __attribute__((visibility("default")))
#else
#define CSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum csa_status {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, misalignment, bad index data found on device */
    CSA_ERR_UNSUPPORTED = 2,  /* valid but outside what the kernels implement (e.g. D % 8 != 0) */
    CSA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    CSA_ERR_TIMEOUT = 4,      /* a bounded device-side wait expired */
    CSA_ERR_WORKSPACE = 5     /* workspace missing or smaller than csa_workspace_size() */
} csa_status;

/* Human-readable name of a status code (static string, never NULL). */
CSA_API const char *csa_status_str(csa_status s);

/* Library version string. */
CSA_API const char *csa_version(void);

/* ---- workspace sizing ------------------------------------------------------------------------ */

typedef enum csa_op {
    CSA_OP_INDEX_TOPK = 1,
    CSA_OP_ATTEND = 2,        /* csa_attend and hca_attend */
    CSA_OP_CSA_FORWARD = 3,
    CSA_OP_HCA_FORWARD = 4,
    CSA_OP_DECODE = 5,
    CSA_OP_HCA_DECODE = 6,    /* hca_decode (B, T, W) */
    CSA_OP_OUT_PROJ = 7       /* csa_out_proj */
} csa_op;

typedef struct csa_dims {
    int64_t S;      /* prefill tokens */
    int64_t T;      /* compressed entries (prefill: floor(S/m); decode: per sequence) */
    int32_t B;      /* decode sequences */
    int32_t H, D;   /* query heads, head dim */
    int32_t HI, dI; /* index heads, index head dim */
    int32_t k;      /* top-k */
    int32_t W;      /* sliding window */
} csa_dims;

/* Bytes of device workspace `op` needs for `dims` (>= 256; the first 256 bytes hold the status word). */
CSA_API size_t csa_workspace_size(csa_op op, const csa_dims *dims);

/* Copies the status word of `workspace` to *status after synchronizing `stream`. */
CSA_API csa_status csa_get_device_status(const void *workspace, int32_t *status, void *stream);

/* ---- 1. compressor ------------------------------------------------------------------------------
 * [HF-V4 "Hybrid attention"; digest]. Entry w pools the window [(w+1)m - L, (w+1)m) clipped at
 * position 0: per channel d, softmax over positions j of gate[j,d] + pos_bias[j - ((w+1)m - L)],
 * weights applied to kv[j,d]. CSA: L = 2m (overlapping), HCA: L = m. The entry is then
 * RoPE-rotated at position w*m with theta_cmp on its last rope_dim channels (interleaved pairs).
 * kv_rot[j] = kv[j] rotated at position j with theta_tok. A chunk at pos0 writes the entries whose
 * window closes inside it, w in [floor(pos0/m), floor((pos0+S)/m)), and kv_rot rows [pos0, pos0+S).
 *   kv, gate   [pos0 + S, D] bf16 by position; rows before max(0, floor(pos0/m)*m + m - L) are not
 *              read (an entry closing in the chunk may pool positions before pos0)
 *   pos_bias   [L] fp32
 *   C          [floor((pos0+S)/m), D] bf16 (out: the chunk's entries; earlier rows untouched)
 *   kv_rot     [pos0 + S, D] bf16 (out: rows [pos0, pos0+S); may be NULL)
 * Requires D % 8 == 0, rope_dim even, rope_dim % 8 == 0, rope_dim <= D, 1 <= m <= L <= 4096,
 * 0 <= pos0 <= 2^40. */
CSA_API csa_status csa_compress(const void *kv, const void *gate, const float *pos_bias,
                        int64_t S, int64_t pos0, int32_t D, int32_t m, int32_t L, int32_t rope_dim,
                        double theta_cmp, double theta_tok,
                        void *C, void *kv_rot, void *stream);

/* ---- 2. lightning indexer + top-k (prefill) ----------------------------------------------------
 * [HF-V4 "Hybrid attention", CSA; "Attention mask layout", CSA layer; digest].
 * For the query at position t = pos0 + i (row i of the chunk):
 * I[t,s] = sum_h w[i,h] * ReLU(qI[i,h,:] . kI[s,:]) for visible entries s < vis(t) = min(T, floor((t+1)/m));
 * idx[i] = the min(k, vis) largest, ties to the smaller s, written in ascending index order,
 * remaining slots -1.
 *   qI [S, HI, dI] bf16   kI [T, dI] bf16 (every entry so far, T <= floor((pos0+S)/m))
 *   w [S, HI] fp32        idx [S, k] int32 (out)
 * Requires dI % 8 == 0, 1 <= k. */
CSA_API csa_status csa_index_topk(const void *qI, const void *kI, const float *w,
                          int64_t S, int64_t pos0, int64_t T, int32_t HI, int32_t dI, int32_t m, int32_t k,
                          int32_t *idx, void *workspace, size_t workspace_bytes, void *stream);

/* ---- 3. sparse + window attention (CSA prefill) ---------------------------------------------
 * [HF-V4 "Hybrid attention": shared K=V MQA, partial interleaved RoPE, output rope slice rotated
 * at -i (eq. 26), per-head sink (eq. 27), sliding-window branch; "Attention mask layout"].
 * For the query at position t = pos0 + i (row i), head h: keys = kv_rot[j] for j in [t-W+1, t]
 * (window) plus C[s] for s in idx[i] (s != -1). Logits lambda*(R_tok(t) q).kv_rot[j] and
 * lambda*(R_cmp(t) q).C[s]; one softmax over all keys plus exp(sinks[h]); K = V; each branch's
 * rope slice rotated back by -t with its theta.
 *   q [S, H, D] bf16 (un-rotated)   C [T, D] bf16 (post-RoPE, T <= floor((pos0+S)/m))
 *   kv_rot [pos0 + S, D] bf16 (post-RoPE, by position)
 *   idx [S, k] int32                sinks [H] fp32               o [S, H, D] fp32 (out)
 * softmax_scale <= 0 selects 1/sqrt(D). Index values >= vis(t) are skipped and reported as
 * CSA_ERR_INVALID_ARG in the workspace status. */
CSA_API csa_status csa_attend(const void *q, const void *C, const void *kv_rot, const int32_t *idx,
                      const float *sinks, int64_t S, int64_t pos0, int32_t H, int32_t D, int64_t T, int32_t k,
                      int32_t W, int32_t rope_dim, int32_t m, double theta_tok, double theta_cmp,
                      float softmax_scale, float *o, void *workspace, size_t workspace_bytes,
                      void *stream);

/* ---- 4. dense compressed + window attention (HCA prefill) --------------------------------------
 * [HF-V4 "Hybrid attention", HCA; "Attention mask layout", HCA layer]. As csa_attend with the
 * entry branch = every visible entry C[w], w < vis(t), t = pos0 + i. */
CSA_API csa_status hca_attend(const void *q, const void *C, const void *kv_rot, const float *sinks,
                      int64_t S, int64_t pos0, int32_t H, int32_t D, int64_t T, int32_t W, int32_t rope_dim,
                      int32_t m, double theta_tok, double theta_cmp, float softmax_scale, float *o,
                      void *workspace, size_t workspace_bytes, void *stream);

/* ---- 5. fused layer forward ----------------------------------------------------------------------
 * csa_forward = csa_compress (L = 2m) -> csa_index_topk -> csa_attend, in stream order.
 * hca_forward = csa_compress (L = m)  -> hca_attend. Intermediates C, kv_rot, idx are
 * caller-provided outputs (kv_rot and C are needed by later decode steps as cache). For a chunk at
 * pos0, kv, gate and kv_rot are [pos0 + S, D] by position, C is [floor((pos0+S)/m), D] holding the
 * earlier chunks' entries, kI [floor((pos0+S)/m), dI] every entry's index key; the rest are the
 * chunk's S rows. */
CSA_API csa_status csa_forward(const void *q, const void *kv, const void *gate, const float *pos_bias,
                       const void *qI, const void *kI, const float *w, const float *sinks,
                       int64_t S, int64_t pos0, int32_t H, int32_t D, int32_t HI, int32_t dI, int32_t m, int32_t L,
                       int32_t k, int32_t W, int32_t rope_dim, double theta_tok, double theta_cmp,
                       float softmax_scale, void *C, void *kv_rot, int32_t *idx, float *o,
                       void *workspace, size_t workspace_bytes, void *stream);

CSA_API csa_status hca_forward(const void *q, const void *kv, const void *gate, const float *pos_bias,
                       const float *sinks, int64_t S, int64_t pos0, int32_t H, int32_t D, int32_t m, int32_t L,
                       int32_t W, int32_t rope_dim, double theta_tok, double theta_cmp,
                       float softmax_scale, void *C, void *kv_rot, float *o,
                       void *workspace, size_t workspace_bytes, void *stream);

/* ---- 6. CSA decode ---------------------------------------------------------------------------------
 * One new query per sequence at position P against post-RoPE caches; every one of the T entries
 * is visible. Indexer + top-k over all T entries, then the attention of csa_attend for row P.
 *   q [B, H, D] bf16 (un-rotated)   qI [B, HI, dI] bf16   w [B, HI] fp32   kI [B, T, dI] bf16
 *   entries: C [B, T, D] bf16, or (C == NULL) the FP8 cache of [digest] as three arrays:
 *            c8 [B, T, D-rope_dim] E4M3 codes, c8_scale [B, T] fp32, c_rope [B, T, rope_dim] bf16;
 *            value = e4m3(c8) * scale on channels [0, D-rope_dim), c_rope on the rest
 *   win [B, W, D] bf16: window rows for positions P-W+1 .. P (rows at negative positions ignored)
 *   sinks [H] fp32    idx_out [B, k] int32 (out, may be NULL)    o [B, H, D] fp32 (out)
 * csa_workspace_size(CSA_OP_DECODE) is the recommended workspace; any workspace down to the index
 * scores, candidates and indices is accepted and uses fewer attention splits per sequence. */
CSA_API csa_status csa_decode(const void *q, const void *qI, const float *w, const void *kI,
                      const void *C, const uint8_t *c8, const float *c8_scale, const void *c_rope,
                      const void *win, const float *sinks, int32_t B, int32_t H, int32_t D,
                      int64_t T, int32_t HI, int32_t dI, int32_t k, int32_t W, int32_t rope_dim,
                      int64_t P, double theta_tok, double theta_cmp, float softmax_scale,
                      int32_t *idx_out, float *o, void *workspace, size_t workspace_bytes,
                      void *stream);

/* ---- 7. CSA decode without caller-provided scratch ---------------------------------------------
 * No counterpart on the source pages: this is a convenience of this library.
 * For callers that cannot allocate device memory (a runtime without its own CUDA allocator, or a
 * serving loop that must not call cudaMalloc while other work is in flight), this is csa_decode
 * with its scratch taken from a fixed 16 MiB array inside the library; every GPU that loads the
 * library holds that array until the process exits. Arguments and results are those of
 * csa_decode, without workspace and workspace_bytes. It allocates nothing.
 *   - Returns CSA_ERR_WORKSPACE, launching nothing, when the problem needs more scratch than the
 *     array holds: the index scores, the top-k histograms, bitmap and candidates, and the selected
 *     indices, about B*(4*T + T/8 + 24 KB + 4*k) bytes (e.g. B=64 sequences of T=32768 entries,
 *     or B=8 of T=262144, fit). Whatever the array has left is used for attention splits.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current; make that first call before any stream capture. The address is kept per
 *     device together with the CUDA context it belongs to and looked up again when a different
 *     context is current (after cudaDeviceReset, or under a context the caller created).
 *   - B, T and k so large that a scratch size would overflow are CSA_ERR_INVALID_ARG.
 *   - All calls on a device share the one array and it keeps the last call's contents: calls that
 *     overlap on the GPU (different streams, or different host threads) race and must be
 *     serialised by the caller. The device status word of the last call is not readable through
 *     csa_get_device_status (there is no workspace pointer to pass). */
CSA_API size_t csa_decode_noalloc_max_scratch(void);

CSA_API csa_status csa_decode_noalloc(const void *q, const void *qI, const float *w, const void *kI,
                      const void *C, const uint8_t *c8, const float *c8_scale, const void *c_rope,
                      const void *win, const float *sinks, int32_t B, int32_t H, int32_t D,
                      int64_t T, int32_t HI, int32_t dI, int32_t k, int32_t W, int32_t rope_dim,
                      int64_t P, double theta_tok, double theta_cmp, float softmax_scale,
                      int32_t *idx_out, float *o, void *stream);

/* ---- 8. HCA decode, and the sliding-window-only layer --------------------------------------------
 * [HF-V4 "Hybrid attention", HCA (dense attention over all pooled entries); "Attention mask layout",
 * HCA layer and sliding-window layer; "Cache layers"].
 * hca_decode: one new query per sequence at position P; keys = every one of the T cached entries
 * (all visible at decode) plus the window rows win[b] (positions P-W+1 .. P), one softmax with the
 * sink; no indexer. Entry caches, window, q, sinks and o as in csa_decode (bf16 C, or the FP8
 * triplet when C == NULL). T = 0 is the decode step of a sliding-window-only layer (window rows and
 * sink only; C may be NULL).
 * csa_workspace_size(CSA_OP_HCA_DECODE) is the recommended workspace (split-K partials over the
 * B*(T+W) keys); any workspace down to 256 bytes is accepted and uses fewer splits. */
CSA_API csa_status hca_decode(const void *q, const void *C, const uint8_t *c8, const float *c8_scale,
                      const void *c_rope, const void *win, const float *sinks, int32_t B, int32_t H,
                      int32_t D, int64_t T, int32_t W, int32_t rope_dim, int64_t P, double theta_tok,
                      double theta_cmp, float softmax_scale, float *o, void *workspace,
                      size_t workspace_bytes, void *stream);

/* swa_attend: prefill of a sliding-window-only layer. For the query at position t = pos0 + i, head h:
 * keys kv_rot[j] for j in [t-W+1, t] (post-RoPE at theta_tok), one softmax with exp(sinks[h]),
 * K = V, the output rope slice rotated back by -t with theta_tok; no compressed entries. Arguments
 * as hca_attend without C, T, m and theta_cmp. Workspace: 256 bytes (the status word). */
CSA_API csa_status swa_attend(const void *q, const void *kv_rot, const float *sinks, int64_t S, int64_t pos0, int32_t H,
                      int32_t D, int32_t W, int32_t rope_dim, double theta_tok, float softmax_scale,
                      float *o, void *workspace, size_t workspace_bytes, void *stream);

/* ---- 9. the compressor's decode step --------------------------------------------------------------
 * [HF-V4 "Hybrid attention" (CSA m-token pooling over overlapping windows, HCA over m'-token
 * windows), "Cache layers" (the compressed buffers carry the tokens of the window still open);
 * digest: softmax gate with a learned position bias, FP8 entries with BF16 rope channels].
 * One new token per sequence at position P (the same P for every sequence; positions start at 0):
 *   x_new [B, D] bf16 (un-rotated kv, or per-token index keys with rope_dim = 0), g_new [B, D] bf16
 *   gate logits, pos_bias [L] fp32. state_x, state_g [B, L, D] bf16 hold the last L tokens
 *   (slot = position mod L); the caller zero-fills nothing: a slot is read only after it was written.
 * The token is written into the state; when (P+1) is a multiple of m, entry w = (P+1)/m - 1 pools
 * positions [(w+1)m - L, (w+1)m) exactly as csa_compress, is rotated at w*m with theta_cmp, and is
 * written to the entry cache: C [B, Tcap, D] bf16, or (C == NULL) the FP8 triplet of csa_decode:
 * c8 [B, Tcap, D - rope_dim] E4M3 codes (8-byte aligned), c8_scale [B, Tcap] = amax/448 over the
 * non-rope channels (1 when they are all zero), c_rope [B, Tcap, rope_dim] bf16. An entry index
 * w >= Tcap is CSA_ERR_INVALID_ARG. With W > 0 the token's row rotated at P with theta_tok is written
 * to win [B, W, D] at slot (W-1-P) mod W, which csa_decode / hca_decode read as the window rows of P.
 * Requires D % 8 == 0, D <= 512. No workspace; stream-ordered. */
CSA_API csa_status csa_compress_append(const void *x_new, const void *g_new, const float *pos_bias,
                      void *state_x, void *state_g, int32_t B, int32_t D, int32_t m, int32_t L,
                      int32_t rope_dim, int64_t P, double theta_cmp, double theta_tok, void *C,
                      uint8_t *c8, float *c8_scale, void *c_rope, int64_t Tcap, void *win, int32_t W,
                      void *stream);

/* ---- 10. grouped low-rank output projection ----------------------------------------------------------
 * [HF-V4 "Hybrid attention", grouped output projection: o_groups head groups, o_lora_rank per group,
 * then hidden_size (o_a_proj as a grouped linear, then o_b_proj); Atlas config: o_groups 8,
 * o_lora_rank 1024, hidden_size 4096].
 *   o   [S, H*D] bf16: the attention output of each token, heads in order (group g = heads
 *       [g H/G, (g+1) H/G), i.e. columns [g K, (g+1) K) with K = (H/G) D)
 *   wa  [G, R, K] bf16: o_a_proj, one [R x K] matrix per group (row = output channel)
 *   wb  [hidden, G*R] bf16: o_b_proj
 *   z   [S, G*R] bf16 (out): z[:, g R + j] = sum_c o[:, g K + c] * wa[g, j, c]
 *   out [S, hidden] bf16 (out): out[:, i] = sum_c z[:, c] * wb[i, c]
 * fp32 accumulation; z is rounded to bf16 before o_b_proj. Requires H % G == 0, R and hidden
 * multiples of 256, K and G*R multiples of 64. Workspace: 256 bytes (the status word). */
CSA_API csa_status csa_out_proj(const void *o, const void *wa, const void *wb, int64_t S, int32_t H, int32_t D,
                      int32_t G, int32_t R, int32_t hidden, void *z, void *out, void *workspace,
                      size_t workspace_bytes, void *stream);

/* ---- 11. FP4 (MXFP4) lightning indexer, prefill and decode ------------------------------------------
 * [Axbrief "Compressed attention and a new optimizer": MXFP4 on the lightning indexer's query-key
 * path; HF-blog digest: the indexer stored in FP4]. MXFP4 is the OCP Microscaling format: blocks of
 * 32 consecutive channels share an E8M0 scale 2^(e-127) (one byte); elements are E2M1 codes (values
 * 0, 0.5, 1, 1.5, 2, 3, 4, 6, sign in bit 3), two per byte, channel 2i in the low nibble.
 *
 * csa_quantize_mxfp4: x [rows, cols] bf16 -> codes [rows, cols/2] uint8, scales [rows, cols/32] uint8.
 *   Per block: amax = max |x|; e = 0 for amax = 0, else clamp(floor(log2 amax) - 2 + 127, 0, 254);
 *   element = x / 2^(e-127) rounded to the nearest E2M1 value, ties to the even code, saturating at 6;
 *   a value that rounds to zero is stored as +0. Requires cols % 32 == 0 and 16-byte aligned x, codes.
 *
 * csa_decode_fp4: csa_decode with the indexer's operands in MXFP4:
 *   qI_codes [B, HI, dI/2], qI_scales [B, HI, dI/32], kI_codes [B, T, dI/2], kI_scales [B, T, dI/32];
 *   the index scores are the indexer formula on the dequantised values (exact products, fp32
 *   accumulation); everything else is csa_decode's. Requires dI of 64 or 128 and HI of 16, 32, 64 or
 *   128; workspace as csa_decode (csa_workspace_size(CSA_OP_DECODE)). With dI = 128, HI <= 64, T a
 *   multiple of 4, 16-byte aligned kI_codes and kI_scales and 4-byte aligned qI_scales the scores come
 *   from the block-scaled tensor-core MMA on the codes as stored; other shapes dequantise each tile to
 *   bf16 in shared memory first (the same scores). */
CSA_API csa_status csa_quantize_mxfp4(const void *x, int64_t rows, int32_t cols, uint8_t *codes, uint8_t *scales,
                              void *stream);

/* csa_index_topk_fp4: csa_index_topk (prefill, chunk at pos0) with the indexer's operands in MXFP4:
 *   qI_codes [S, HI, dI/2], qI_scales [S, HI, dI/32], kI_codes [T, dI/2], kI_scales [T, dI/32]
 *   (layout of csa_quantize_mxfp4); w [S, HI] fp32; idx [S, k] int32 (out).
 * The scores are the indexer formula on the dequantised values (exact products, fp32 accumulation),
 * computed by the block-scaled tensor-core MMA; the top-k is csa_index_topk's. Requires dI = 128,
 * HI of 16, 32 or 64, T <= 4096, 16-byte aligned codes and 4-byte aligned scales. Workspace: 256 bytes
 * (the status word). */
CSA_API csa_status csa_index_topk_fp4(const uint8_t *qI_codes, const uint8_t *qI_scales, const float *w,
                              const uint8_t *kI_codes, const uint8_t *kI_scales, int64_t S, int64_t pos0, int64_t T,
                              int32_t HI, int32_t dI, int32_t m, int32_t k, int32_t *idx, void *workspace,
                              size_t workspace_bytes, void *stream);

CSA_API csa_status csa_decode_fp4(const void *q, const uint8_t *qI_codes, const uint8_t *qI_scales, const float *w,
                      const uint8_t *kI_codes, const uint8_t *kI_scales, const void *C, const uint8_t *c8,
                      const float *c8_scale, const void *c_rope, const void *win, const float *sinks, int32_t B,
                      int32_t H, int32_t D, int64_t T, int32_t HI, int32_t dI, int32_t k, int32_t W,
                      int32_t rope_dim, int64_t P, double theta_tok, double theta_cmp, float softmax_scale,
                      int32_t *idx_out, float *o, void *workspace, size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* CSA_B200_H */
