// kernels.cuh -- launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace csa {

// Arguments of the attention kernels (prefill rows or decode sequences).
struct AttnArgs {
    const uint16_t *q;         // [R, H, D] bf16, un-rotated
    const uint16_t *win;       // prefill: kv_rot [S, D]; decode: win [R, W, D] (post-RoPE)
    const uint16_t *C;         // bf16 entries: prefill [T, D]; decode [R, T, D] (or null = fp8 cache)
    const uint8_t *c8;         // fp8 entries [R, T, D-r]
    const float *c8_scale;     // [R, T]
    const uint16_t *c_rope;    // [R, T, r]
    const int32_t *idx;        // [R, k] or null (all visible entries: HCA)
    const float *sinks;        // [H]
    float *o;                  // [R, H, D] fp32
    int32_t *status;           // workspace status word
    int64_t R, T, P;           // rows, entries (per row for decode), decode position
    int64_t pos0;              // prefill: position of row 0 (kv_rot rows are absolute positions)
    int H, D, k, W, r, m, decode;
    int after_kernel;          // launch as a programmatic dependent of the kernel before it in the stream
    float scale;
    double log2_theta_tok, log2_theta_cmp;
};

// compress.cu: one prefill chunk at positions [pos0, pos0 + S): entries [floor(pos0/m), floor((pos0+S)/m))
// into C and rows [pos0, pos0 + S) into kv_rot (either may be null); kv, gate, C, kv_rot by absolute index
cudaError_t launch_compress(const uint16_t *kv, const uint16_t *gate, const float *bias, int64_t S, int64_t pos0,
                            int D, int m, int L, int r, double theta_cmp, double theta_tok, uint16_t *C,
                            uint16_t *kv_rot, cudaStream_t stream);
// index_topk.cu: general-path scores and top-k; prefill row r is the query at position pos0 + r
cudaError_t launch_index_scores(const uint16_t *qI, const float *w, const uint16_t *kI, int64_t R, int64_t pos0,
                                int64_t T, int HI, int dI, int m, int decode, float *scores, cudaStream_t stream);
cudaError_t launch_topk_rows(const float *scores, int64_t R, int64_t pos0, int64_t T, int m, int decode, int k,
                             int32_t *idx, cudaStream_t stream);
cudaError_t launch_attend_simt(const AttnArgs &a, cudaStream_t stream);

// attend_tc.cu: tcgen05 prefill attention for H=64, D=512, rope 64 (CSA when idx != null, else HCA)
bool attend_tc_supported(int H, int D, int r, int k);
cudaError_t launch_attend_tc(const AttnArgs &a, cudaStream_t stream);
// decode: nsplit CTAs per sequence with partials in `part` (attend_tc_decode_partials bytes) + combine
size_t attend_tc_decode_partials(int64_t B, int nsplit);
cudaError_t launch_attend_tc_decode(const AttnArgs &a, int nsplit, float *part, cudaStream_t stream);

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, box [box_rows, 64], 128-byte swizzle
bool make_tmap_bf16_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// 2-D fp32 tensor map, box [box_rows, 32], 128-byte swizzle
bool make_tmap_f32_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// 2-D byte tensor map over [rows, cols] (cols a multiple of 16, at most 256), box [box_rows, cols], no swizzle
bool make_tmap_u8_rows(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// 2-D byte tensor map over [rows, 64], box [box_rows, 64], 64-byte swizzle
bool make_tmap_u8_sw64(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows);
// [rows, 64] bytes as 128-row boxes whose shared-memory row 32 j + r is source row 4 r + j, 64-byte swizzle

// append.cu: the compressor's decode step (one token per sequence; emits an entry when a window closes)
struct AppendArgs {
    const uint16_t *x_new, *g_new;   // [B, D] bf16 token at position P and its gate logits
    const float *bias;               // [L] position bias of the pooling window
    uint16_t *state_x, *state_g;     // [B, L, D] bf16 rings of the last L tokens (slot = position mod L)
    uint16_t *C;                     // [B, Tcap, D] bf16 entry cache, or null for the FP8 cache:
    uint8_t *c8;                     //   [B, Tcap, D - r] E4M3 codes
    float *c8_scale;                 //   [B, Tcap]
    uint16_t *c_rope;                //   [B, Tcap, r] bf16 rope channels
    uint16_t *win;                   // [B, W, D] window ring (slot (W-1-P) mod W), or null
    int64_t P, Tcap;
    int B, D, m, L, r, W;
    double log2_theta_cmp, log2_theta_tok;
};
cudaError_t launch_compress_append(const AppendArgs &a, cudaStream_t stream);

// proj.cu: grouped GEMM C[:, gN:(g+1)N] = A[:, gK:(g+1)K] . B[gN:(g+1)N, :]^T (bf16, fp32 accumulate)
bool proj_gemm_tc_supported(int64_t M, int N, int K, int G);
cudaError_t launch_proj_gemm_tc(const uint16_t *A, int64_t lda, const uint16_t *B, uint16_t *C, int64_t ldc, int64_t M,
                                int N, int K, int G, int32_t *status, cudaStream_t stream);

// api.cu: smallest workspace csa_decode accepts (no attention split partials)
size_t decode_workspace_min(int64_t B, int64_t T, int32_t k);
// api.cu: false when B, T or k are so large that a decode workspace size would overflow size_t
bool decode_sizes_representable(int64_t B, int64_t T, int32_t k);

// decode_tc.cu: decode index scan (tcgen05, HBM streaming) + two-stage exact top-k
size_t decode_index_workspace(int64_t B, int64_t T, int k);
size_t decode_index_head_bytes(int64_t B);   // leading bytes of its workspace the caller zeroes
bool decode_index_tc_supported(int64_t T, int HI, int dI, int k);
cudaError_t launch_decode_index_tc(const uint16_t *qI, const float *w, const uint16_t *kI, int64_t B, int64_t T, int HI,
                                   int dI, int k, int32_t *idx, void *ws, int32_t *status, cudaStream_t stream);
// the same on MXFP4 q^I and k^I (codes two per byte, one E8M0 scale per 32 channels)
bool decode_index_fp4_supported(int64_t T, int HI, int dI, int k);
cudaError_t launch_decode_index_fp4(const uint8_t *qc, const uint8_t *qs, const float *w, const uint8_t *kc,
                                    const uint8_t *ks, int64_t B, int64_t T, int HI, int dI, int k, int32_t *idx,
                                    void *ws, int32_t *status, cudaStream_t stream);
// fp4.cu: bf16 rows -> MXFP4 codes and scales
cudaError_t launch_quantize_mxfp4(const uint16_t *x, int64_t rows, int cols, uint8_t *codes, uint8_t *scales,
                                  cudaStream_t stream);

// index_tc.cu: tcgen05 indexer with fused top-k (entries on TMEM lanes, scores kept on chip)
bool index_topk_tc_supported(int64_t T, int HI, int dI, int k);
cudaError_t launch_index_topk_tc(const uint16_t *qI, const uint16_t *kI, const float *w, int64_t S, int64_t pos0,
                                 int64_t T, int HI, int dI, int m, int k, int32_t *idx, int32_t *status,
                                 cudaStream_t stream);
// the same on MXFP4 q^I and k^I (d_I = 128, HI <= 64): block-scaled MMA, fused top-k
bool index_topk_fp4_supported(int64_t T, int HI, int dI, int k);
cudaError_t launch_index_topk_fp4(const uint8_t *qc, const uint8_t *qs, const float *w, const uint8_t *kc,
                                  const uint8_t *ks, int64_t S, int64_t pos0, int64_t T, int HI, int dI, int m, int k,
                                  int32_t *idx, int32_t *status, cudaStream_t stream);

}  // namespace csa
