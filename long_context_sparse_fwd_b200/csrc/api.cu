// api.cu -- the C ABI declared in include/csa.h: host-side argument checks, workspace layout and
// launch sequencing. Nothing here allocates device memory; every buffer is the caller's.
#include <math.h>
#include <algorithm>
#include <string.h>

#include "kernels.cuh"


using namespace csa;

namespace {

constexpr size_t kStatusBytes = 256;

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }

inline csa_status from_cuda(cudaError_t e)
{
    return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}

#define CSA_CHECK_ARG(cond)                \
    do {                                   \
        if (!(cond)) return CSA_ERR_INVALID_ARG; \
    } while (0)
#define CSA_CHECK_SUP(cond)                \
    do {                                   \
        if (!(cond)) return CSA_ERR_UNSUPPORTED; \
    } while (0)
#define CSA_TRY(expr)                                   \
    do {                                                \
        csa_status _s = (expr);                         \
        if (_s != CSA_OK) return _s;                    \
    } while (0)
#define CSA_CUDA(expr)                                  \
    do {                                                \
        if ((expr) != cudaSuccess) return CSA_ERR_CUDA; \
    } while (0)

inline bool theta_ok(double th) { return isfinite(th) && th > 1.0; }

size_t scores_bytes(int64_t R, int64_t T) { return align256(sizeof(float) * (size_t)R * (size_t)T); }

csa_status check_workspace(void *ws, size_t bytes, size_t need)
{
    if (ws == nullptr || bytes < need) return CSA_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return CSA_ERR_INVALID_ARG;
    return CSA_OK;
}

csa_status reset_status(void *ws, cudaStream_t stream)
{
    CSA_CUDA(cudaMemsetAsync(ws, 0, sizeof(int32_t), stream));
    return CSA_OK;
}

csa_status check_compress(const void *kv, const void *gate, const float *pos_bias, int64_t S, int64_t pos0,
                          int32_t D, int32_t m, int32_t L, int32_t r, double theta_cmp, double theta_tok, const void *C)
{
    CSA_CHECK_ARG(S >= 0 && pos0 >= 0 && pos0 <= ((int64_t)1 << 40) && D > 0 && m >= 1 && L >= m && r >= 0 &&
                  r <= D && (r % 2) == 0);
    CSA_CHECK_ARG(S == 0 || (kv != nullptr && gate != nullptr && pos_bias != nullptr));
    CSA_CHECK_ARG((pos0 + S) / m == pos0 / m || C != nullptr);   // entries close in this chunk
    CSA_CHECK_ARG(r == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_SUP(D % 8 == 0 && r % 8 == 0 && L <= 4096);
    CSA_CHECK_ARG(aligned16(kv) && aligned16(gate) && aligned16(C));
    return CSA_OK;
}

csa_status check_attend_common(const void *q, const void *C, const void *kv_rot, const float *sinks, int64_t S,
                               int64_t pos0, int32_t H, int32_t D, int64_t T, int32_t W, int32_t r, int32_t m,
                               double theta_tok, double theta_cmp, const float *o)
{
    CSA_CHECK_ARG(S >= 0 && pos0 >= 0 && pos0 <= ((int64_t)1 << 40) && H > 0 && D > 0 && T >= 0 && W >= 0 &&
                  m >= 1 && r >= 0 && r <= D && (r % 2) == 0);
    CSA_CHECK_ARG(T <= (pos0 + S) / m);
    CSA_CHECK_ARG(S == 0 || (q != nullptr && sinks != nullptr && o != nullptr));
    CSA_CHECK_ARG(S == 0 || W == 0 || kv_rot != nullptr);
    CSA_CHECK_ARG(T == 0 || C != nullptr);
    CSA_CHECK_ARG(r == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_SUP(D == 64 || D == 128 || D == 256 || D == 512);
    CSA_CHECK_SUP(r % 8 == 0);
    CSA_CHECK_ARG(aligned16(q) && aligned16(C) && aligned16(kv_rot) && aligned16(o));
    return CSA_OK;
}

AttnArgs prefill_args(const void *q, const void *C, const void *kv_rot, const int32_t *idx, const float *sinks,
                      int64_t S, int64_t pos0, int32_t H, int32_t D, int64_t T, int32_t k, int32_t W, int32_t r,
                      int32_t m, double theta_tok, double theta_cmp, float scale, float *o, void *ws)
{
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const uint16_t *>(q);
    a.win = static_cast<const uint16_t *>(kv_rot);
    a.C = static_cast<const uint16_t *>(C);
    a.idx = idx;
    a.sinks = sinks;
    a.o = o;
    a.status = static_cast<int32_t *>(ws);
    a.R = S;
    a.pos0 = pos0;
    a.T = T;
    a.H = H;
    a.D = D;
    a.k = k;
    a.W = W;
    a.r = r;
    a.m = m;
    a.scale = scale > 0.f ? scale : (float)(1.0 / sqrt((double)D));
    a.log2_theta_tok = r > 0 ? log2(theta_tok) : 0.0;
    a.log2_theta_cmp = r > 0 ? log2(theta_cmp) : 0.0;
    return a;
}

// Decode workspace: status word, index scores/candidates, selected indices, then the attention
// split partials (optional: fewer splits when the workspace is smaller).
size_t decode_index_bytes(int64_t B, int64_t T, int32_t k)
{
    return align256(std::max(scores_bytes(B, T), decode_index_workspace(B, T, k)));
}

// attention CTAs per sequence: about one wave of CTAs over the SMs (one CTA fits per SM)
int decode_splits_preferred(int64_t B)
{
    return (int)std::min<int64_t>(8, std::max<int64_t>(1, 148 / std::max<int64_t>(B, 1)));
}

// HCA decode: up to 16 splits per sequence (about one wave of CTAs), never more than its key blocks
int hca_decode_splits_preferred(int64_t B, int64_t T, int32_t W)
{
    const int64_t blocks = (T + 63) / 64 + ((int64_t)std::max(W, 0) + 63) / 64;
    const int64_t by_sm = std::max<int64_t>(1, 148 / std::max<int64_t>(B, 1));
    return (int)std::max<int64_t>(1, std::min<int64_t>(std::min<int64_t>(16, by_sm), std::max<int64_t>(blocks, 1)));
}

}  // namespace

namespace csa {
// Every decode workspace term is at most a few times 4*B*T or 4*B*k bytes: with T <= 2^40 entries
// per sequence and B*T, B*k below 2^56 none of them can overflow a 64-bit size.
bool decode_sizes_representable(int64_t B, int64_t T, int32_t k)
{
    if (B < 0 || T < 0 || k < 0 || T > ((int64_t)1 << 40)) return false;
    const uint64_t lim = (uint64_t)1 << 56;
    return B == 0 || ((uint64_t)T <= lim / (uint64_t)B && (uint64_t)k <= lim / (uint64_t)B);
}

size_t decode_workspace_min(int64_t B, int64_t T, int32_t k)
{
    return kStatusBytes + decode_index_bytes(B, T, k) + align256(sizeof(int32_t) * (size_t)B * (size_t)k);
}
}  // namespace csa

namespace {

// Prefill attention: the tcgen05 kernel for the V4 head shape (64 heads x 512, rope 64), else the
// general CUDA-core kernel.
cudaError_t attend_any(const AttnArgs &a, cudaStream_t st)
{
    if (!a.decode && attend_tc_supported(a.H, a.D, a.r, a.idx != nullptr ? a.k : 0)) return launch_attend_tc(a, st);
    return launch_attend_simt(a, st);
}

// Prefill indexer + top-k: the tcgen05 kernel with on-chip scores where it applies, else the
// general path (scores through the workspace, then a radix select per row).
cudaError_t index_topk_any(const void *qI, const void *kI, const float *w, int64_t S, int64_t pos0, int64_t T,
                           int32_t HI, int32_t dI, int32_t m, int32_t k, int32_t *idx, void *workspace, cudaStream_t st)
{
    const uint16_t *q16 = static_cast<const uint16_t *>(qI), *k16 = static_cast<const uint16_t *>(kI);
    if (T > 0 && index_topk_tc_supported(T, HI, dI, k))
        return launch_index_topk_tc(q16, k16, w, S, pos0, T, HI, dI, m, k, idx, static_cast<int32_t *>(workspace), st);
    float *scores = reinterpret_cast<float *>(static_cast<char *>(workspace) + kStatusBytes);
    cudaError_t e = launch_index_scores(q16, w, k16, S, pos0, T, HI, dI, m, 0, scores, st);
    if (e != cudaSuccess) return e;
    return launch_topk_rows(scores, S, pos0, T, m, 0, k, idx, st);
}

}  // namespace

extern "C" {

const char *csa_status_str(csa_status s)
{
    switch (s) {
    case CSA_OK: return "CSA_OK";
    case CSA_ERR_INVALID_ARG: return "CSA_ERR_INVALID_ARG";
    case CSA_ERR_UNSUPPORTED: return "CSA_ERR_UNSUPPORTED";
    case CSA_ERR_CUDA: return "CSA_ERR_CUDA";
    case CSA_ERR_TIMEOUT: return "CSA_ERR_TIMEOUT";
    case CSA_ERR_WORKSPACE: return "CSA_ERR_WORKSPACE";
    }
    return "CSA_ERR_UNKNOWN";
}

const char *csa_version(void) { return "csa-b200 0.1 (sm_100a)"; }

size_t csa_workspace_size(csa_op op, const csa_dims *d)
{
    if (d == nullptr) return 0;
    switch (op) {
    case CSA_OP_INDEX_TOPK:
    case CSA_OP_CSA_FORWARD:
        // the tensor-core indexer keeps its scores on chip; the general path stages S x T scores.
        // Without the index shape (HI = 0) the general path's size is returned.
        if (d->HI > 0 && d->T > 0 && index_topk_tc_supported(d->T, d->HI, d->dI, std::max(d->k, 1))) return kStatusBytes;
        return kStatusBytes + scores_bytes(d->S, d->T);
    case CSA_OP_ATTEND:
    case CSA_OP_HCA_FORWARD:
        return kStatusBytes;
    case CSA_OP_DECODE:
        return decode_workspace_min(d->B, d->T, d->k) +
               align256(attend_tc_decode_partials(d->B, decode_splits_preferred(d->B)));
    case CSA_OP_HCA_DECODE:
        return kStatusBytes + align256(attend_tc_decode_partials(d->B, hca_decode_splits_preferred(d->B, d->T, d->W)));
    case CSA_OP_OUT_PROJ:
        return kStatusBytes;
    }
    return 0;
}

csa_status csa_get_device_status(const void *workspace, int32_t *status, void *stream)
{
    CSA_CHECK_ARG(workspace != nullptr && status != nullptr);
    int32_t v = 0;
    CSA_CUDA(cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, as_stream(stream)));
    CSA_CUDA(cudaStreamSynchronize(as_stream(stream)));
    *status = v;
    return CSA_OK;
}

csa_status csa_compress(const void *kv, const void *gate, const float *pos_bias, int64_t S, int64_t pos0, int32_t D,
                        int32_t m, int32_t L, int32_t rope_dim, double theta_cmp, double theta_tok, void *C,
                        void *kv_rot, void *stream)
{
    CSA_TRY(check_compress(kv, gate, pos_bias, S, pos0, D, m, L, rope_dim, theta_cmp, theta_tok, C));
    CSA_CHECK_ARG(aligned16(kv_rot));
    return from_cuda(launch_compress(static_cast<const uint16_t *>(kv), static_cast<const uint16_t *>(gate),
                                     pos_bias, S, pos0, D, m, L, rope_dim, theta_cmp, theta_tok,
                                     static_cast<uint16_t *>(C), static_cast<uint16_t *>(kv_rot), as_stream(stream)));
}

csa_status csa_index_topk(const void *qI, const void *kI, const float *w, int64_t S, int64_t pos0, int64_t T,
                          int32_t HI, int32_t dI, int32_t m, int32_t k, int32_t *idx, void *workspace,
                          size_t workspace_bytes, void *stream)
{
    CSA_CHECK_ARG(S >= 0 && pos0 >= 0 && pos0 <= ((int64_t)1 << 40) && T >= 0 && HI > 0 && dI > 0 && m >= 1 && k >= 1);
    CSA_CHECK_ARG(T <= (pos0 + S) / m);
    CSA_CHECK_ARG(S == 0 || (qI != nullptr && w != nullptr && idx != nullptr));
    CSA_CHECK_ARG(T == 0 || kI != nullptr);
    CSA_CHECK_SUP(dI == 32 || dI == 64 || dI == 128 || dI == 256);
    CSA_CHECK_SUP(HI <= 128 && (size_t)HI * dI * 4 <= 160 * 1024);
    CSA_CHECK_ARG(aligned16(qI) && aligned16(kI));
    csa_dims dims;
    memset(&dims, 0, sizeof dims);
    dims.S = S;
    dims.T = T;
    dims.HI = HI;
    dims.dI = dI;
    dims.k = k;
    CSA_TRY(check_workspace(workspace, workspace_bytes, csa_workspace_size(CSA_OP_INDEX_TOPK, &dims)));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    CSA_CUDA(index_topk_any(qI, kI, w, S, pos0, T, HI, dI, m, k, idx, workspace, st));
    return CSA_OK;
}

csa_status csa_attend(const void *q, const void *C, const void *kv_rot, const int32_t *idx, const float *sinks,
                      int64_t S, int64_t pos0, int32_t H, int32_t D, int64_t T, int32_t k, int32_t W, int32_t rope_dim,
                      int32_t m, double theta_tok, double theta_cmp, float softmax_scale, float *o, void *workspace,
                      size_t workspace_bytes, void *stream)
{
    CSA_TRY(check_attend_common(q, C, kv_rot, sinks, S, pos0, H, D, T, W, rope_dim, m, theta_tok, theta_cmp, o));
    CSA_CHECK_ARG(k >= 1 && (S == 0 || idx != nullptr));
    CSA_CHECK_SUP(k <= 4096);
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    AttnArgs a = prefill_args(q, C, kv_rot, idx, sinks, S, pos0, H, D, T, k, W, rope_dim, m, theta_tok, theta_cmp,
                              softmax_scale, o, workspace);
    return from_cuda(attend_any(a, st));
}

csa_status hca_attend(const void *q, const void *C, const void *kv_rot, const float *sinks, int64_t S, int64_t pos0,
                      int32_t H, int32_t D, int64_t T, int32_t W, int32_t rope_dim, int32_t m, double theta_tok,
                      double theta_cmp, float softmax_scale, float *o, void *workspace, size_t workspace_bytes,
                      void *stream)
{
    CSA_TRY(check_attend_common(q, C, kv_rot, sinks, S, pos0, H, D, T, W, rope_dim, m, theta_tok, theta_cmp, o));
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    AttnArgs a = prefill_args(q, C, kv_rot, nullptr, sinks, S, pos0, H, D, T, 0, W, rope_dim, m, theta_tok, theta_cmp,
                              softmax_scale, o, workspace);
    return from_cuda(attend_any(a, st));
}

csa_status csa_forward(const void *q, const void *kv, const void *gate, const float *pos_bias, const void *qI,
                       const void *kI, const float *w, const float *sinks, int64_t S, int64_t pos0, int32_t H,
                       int32_t D, int32_t HI, int32_t dI, int32_t m, int32_t L, int32_t k, int32_t W, int32_t rope_dim,
                       double theta_tok, double theta_cmp, float softmax_scale, void *C, void *kv_rot, int32_t *idx,
                       float *o, void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_TRY(check_compress(kv, gate, pos_bias, S, pos0, D, m, L, rope_dim, theta_cmp, theta_tok, C));
    const int64_t T = (pos0 + S) / m;
    CSA_CHECK_ARG(kv_rot != nullptr || S == 0);
    CSA_TRY(check_attend_common(q, C, kv_rot, sinks, S, pos0, H, D, T, W, rope_dim, m, theta_tok, theta_cmp, o));
    CSA_CHECK_ARG(k >= 1 && (S == 0 || idx != nullptr));
    CSA_CHECK_SUP(k <= 4096);
    CSA_CHECK_ARG(HI > 0 && dI > 0 && (S == 0 || (qI != nullptr && w != nullptr)) && (T == 0 || kI != nullptr));
    CSA_CHECK_SUP(dI == 32 || dI == 64 || dI == 128 || dI == 256);
    CSA_CHECK_SUP(HI <= 128 && (size_t)HI * dI * 4 <= 160 * 1024);
    CSA_CHECK_ARG(aligned16(qI) && aligned16(kI) && aligned16(kv_rot));
    csa_dims dims;
    memset(&dims, 0, sizeof dims);
    dims.S = S;
    dims.T = T;
    dims.HI = HI;
    dims.dI = dI;
    dims.k = k;
    CSA_TRY(check_workspace(workspace, workspace_bytes, csa_workspace_size(CSA_OP_CSA_FORWARD, &dims)));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    CSA_CUDA(launch_compress(static_cast<const uint16_t *>(kv), static_cast<const uint16_t *>(gate), pos_bias, S, pos0,
                             D, m, L, rope_dim, theta_cmp, theta_tok, static_cast<uint16_t *>(C),
                             static_cast<uint16_t *>(kv_rot), st));
    CSA_CUDA(index_topk_any(qI, kI, w, S, pos0, T, HI, dI, m, k, idx, workspace, st));
    AttnArgs a = prefill_args(q, C, kv_rot, idx, sinks, S, pos0, H, D, T, k, W, rope_dim, m, theta_tok, theta_cmp,
                              softmax_scale, o, workspace);
    return from_cuda(attend_any(a, st));
}

csa_status hca_forward(const void *q, const void *kv, const void *gate, const float *pos_bias, const float *sinks,
                       int64_t S, int64_t pos0, int32_t H, int32_t D, int32_t m, int32_t L, int32_t W,
                       int32_t rope_dim, double theta_tok, double theta_cmp, float softmax_scale, void *C, void *kv_rot,
                       float *o, void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_TRY(check_compress(kv, gate, pos_bias, S, pos0, D, m, L, rope_dim, theta_cmp, theta_tok, C));
    const int64_t T = (pos0 + S) / m;
    CSA_CHECK_ARG(kv_rot != nullptr || S == 0);
    CSA_TRY(check_attend_common(q, C, kv_rot, sinks, S, pos0, H, D, T, W, rope_dim, m, theta_tok, theta_cmp, o));
    CSA_CHECK_ARG(aligned16(kv_rot));
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    CSA_CUDA(launch_compress(static_cast<const uint16_t *>(kv), static_cast<const uint16_t *>(gate), pos_bias, S, pos0,
                             D, m, L, rope_dim, theta_cmp, theta_tok, static_cast<uint16_t *>(C),
                             static_cast<uint16_t *>(kv_rot), st));
    AttnArgs a = prefill_args(q, C, kv_rot, nullptr, sinks, S, pos0, H, D, T, 0, W, rope_dim, m, theta_tok, theta_cmp,
                              softmax_scale, o, workspace);
    return from_cuda(attend_any(a, st));
}

// The attention of a decode step once the index lists `idx` are on the stream (shared by csa_decode
// and csa_decode_fp4).
static csa_status decode_attention(const void *q, const void *C, const uint8_t *c8, const float *c8_scale,
                                   const void *c_rope, const void *win, const float *sinks, int32_t B, int32_t H,
                                   int32_t D, int64_t T, int32_t k, int32_t W, int32_t rope_dim, int64_t P,
                                   double theta_tok, double theta_cmp, float softmax_scale, int32_t *idx, float *o,
                                   void *workspace, size_t workspace_bytes, cudaStream_t st)
{
    char *base = static_cast<char *>(workspace);
    const size_t used = decode_workspace_min(B, T, k);
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const uint16_t *>(q);
    a.win = static_cast<const uint16_t *>(win);
    a.C = static_cast<const uint16_t *>(C);
    a.c8 = c8;
    a.c8_scale = c8_scale;
    a.c_rope = static_cast<const uint16_t *>(c_rope);
    a.idx = idx;
    a.sinks = sinks;
    a.o = o;
    a.status = static_cast<int32_t *>(workspace);
    a.R = B;
    a.T = T;
    a.P = P;
    a.H = H;
    a.D = D;
    a.k = k;
    a.W = W;
    a.r = rope_dim;
    a.m = 1;
    a.decode = 1;
    a.after_kernel = 1;   // the top-k kernel precedes it on the stream
    a.scale = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / sqrt((double)D));
    a.log2_theta_tok = rope_dim > 0 ? log2(theta_tok) : 0.0;
    a.log2_theta_cmp = rope_dim > 0 ? log2(theta_cmp) : 0.0;
    if (attend_tc_supported(H, D, rope_dim, k)) {
        // as many attention splits per sequence as the workspace holds (up to the preferred count)
        int nsplit = decode_splits_preferred(B);
        while (nsplit > 1 && used + align256(attend_tc_decode_partials(B, nsplit)) > workspace_bytes) --nsplit;
        return from_cuda(launch_attend_tc_decode(a, nsplit, reinterpret_cast<float *>(base + used), st));
    }
    return from_cuda(launch_attend_simt(a, st));
}

csa_status csa_decode(const void *q, const void *qI, const float *w, const void *kI, const void *C, const uint8_t *c8,
                      const float *c8_scale, const void *c_rope, const void *win, const float *sinks, int32_t B,
                      int32_t H, int32_t D, int64_t T, int32_t HI, int32_t dI, int32_t k, int32_t W, int32_t rope_dim,
                      int64_t P, double theta_tok, double theta_cmp, float softmax_scale, int32_t *idx_out, float *o,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_CHECK_ARG(B >= 0 && H > 0 && D > 0 && T >= 0 && HI > 0 && dI > 0 && k >= 1 && W >= 0 && P >= 0);
    CSA_CHECK_ARG(decode_sizes_representable(B, T, k));
    CSA_CHECK_ARG(rope_dim >= 0 && rope_dim <= D && (rope_dim % 2) == 0);
    CSA_CHECK_ARG(rope_dim == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_ARG(B == 0 || (q != nullptr && qI != nullptr && w != nullptr && sinks != nullptr && o != nullptr));
    CSA_CHECK_ARG(B == 0 || T == 0 || kI != nullptr);
    CSA_CHECK_ARG(B == 0 || W == 0 || win != nullptr);
    const bool fp8 = C == nullptr;
    CSA_CHECK_ARG(B == 0 || T == 0 || !fp8 || (c8 != nullptr && c8_scale != nullptr && c_rope != nullptr));
    CSA_CHECK_SUP(D == 64 || D == 128 || D == 256 || D == 512);
    CSA_CHECK_SUP(rope_dim % 8 == 0 && k <= 4096);
    CSA_CHECK_SUP(dI == 32 || dI == 64 || dI == 128 || dI == 256);
    CSA_CHECK_SUP(HI <= 128 && (size_t)HI * dI * 4 <= 160 * 1024);
    CSA_CHECK_ARG(aligned16(q) && aligned16(qI) && aligned16(kI) && aligned16(C) && aligned16(c8) &&
                  aligned16(c_rope) && aligned16(win) && aligned16(o));
    csa_dims dims;
    memset(&dims, 0, sizeof dims);
    dims.B = B;
    dims.T = T;
    dims.k = k;
    CSA_TRY(check_workspace(workspace, workspace_bytes, decode_workspace_min(B, T, k)));
    cudaStream_t st = as_stream(stream);
    char *base = static_cast<char *>(workspace);
    float *scores = reinterpret_cast<float *>(base + kStatusBytes);
    const size_t index_ws = decode_index_bytes(B, T, k);
    int32_t *idx = idx_out != nullptr ? idx_out : reinterpret_cast<int32_t *>(base + kStatusBytes + index_ws);
    if (T > 0 && decode_index_tc_supported(T, HI, dI, k)) {
        // one clear: the status word and the head of the index workspace that follows it
        CSA_CUDA(cudaMemsetAsync(workspace, 0, kStatusBytes + decode_index_head_bytes(B), st));
        CSA_CUDA(launch_decode_index_tc(static_cast<const uint16_t *>(qI), w, static_cast<const uint16_t *>(kI), B, T,
                                        HI, dI, k, idx, scores, static_cast<int32_t *>(workspace), st));
    } else {
        CSA_TRY(reset_status(workspace, st));
        CSA_CUDA(launch_index_scores(static_cast<const uint16_t *>(qI), w, static_cast<const uint16_t *>(kI), B, 0, T,
                                     HI, dI, 1, 1, scores, st));
        CSA_CUDA(launch_topk_rows(scores, B, 0, T, 1, 1, k, idx, st));
    }
    return decode_attention(q, C, c8, c8_scale, c_rope, win, sinks, B, H, D, T, k, W, rope_dim, P, theta_tok, theta_cmp,
                            softmax_scale, idx, o, workspace, workspace_bytes, st);
}

csa_status csa_quantize_mxfp4(const void *x, int64_t rows, int32_t cols, uint8_t *codes, uint8_t *scales, void *stream)
{
    CSA_CHECK_ARG(rows >= 0 && cols > 0 && cols % 32 == 0);
    CSA_CHECK_ARG(rows == 0 || (x != nullptr && codes != nullptr && scales != nullptr));
    CSA_CHECK_ARG(aligned16(x) && aligned16(codes));
    return from_cuda(launch_quantize_mxfp4(static_cast<const uint16_t *>(x), rows, cols, codes, scales,
                                           as_stream(stream)));
}

csa_status csa_index_topk_fp4(const uint8_t *qI_codes, const uint8_t *qI_scales, const float *w, const uint8_t *kI_codes,
                              const uint8_t *kI_scales, int64_t S, int64_t pos0, int64_t T, int32_t HI, int32_t dI,
                              int32_t m, int32_t k, int32_t *idx, void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_CHECK_ARG(S >= 0 && pos0 >= 0 && pos0 <= ((int64_t)1 << 40) && T >= 0 && HI > 0 && dI > 0 && m >= 1 && k >= 1);
    CSA_CHECK_ARG(T <= (pos0 + S) / m);
    CSA_CHECK_ARG(S == 0 || (qI_codes != nullptr && qI_scales != nullptr && w != nullptr && idx != nullptr));
    CSA_CHECK_ARG(T == 0 || (kI_codes != nullptr && kI_scales != nullptr));
    CSA_CHECK_ARG(aligned16(qI_codes) && aligned16(kI_codes) && (reinterpret_cast<uintptr_t>(qI_scales) & 3u) == 0 &&
                  (reinterpret_cast<uintptr_t>(kI_scales) & 3u) == 0);
    CSA_CHECK_SUP(dI == 128 && (HI == 16 || HI == 32 || HI == 64) && T <= 4096);
    CSA_CHECK_SUP(T == 0 || index_topk_fp4_supported(T, HI, dI, k));
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    if (T == 0) {   // nothing visible yet: every slot is -1
        float *none = nullptr;
        CSA_CUDA(launch_topk_rows(none, S, pos0, 0, m, 0, k, idx, st));
        return CSA_OK;
    }
    CSA_CUDA(launch_index_topk_fp4(qI_codes, qI_scales, w, kI_codes, kI_scales, S, pos0, T, HI, dI, m, k, idx,
                                   static_cast<int32_t *>(workspace), st));
    return CSA_OK;
}

csa_status csa_decode_fp4(const void *q, const uint8_t *qI_codes, const uint8_t *qI_scales, const float *w,
                          const uint8_t *kI_codes, const uint8_t *kI_scales, const void *C, const uint8_t *c8,
                          const float *c8_scale, const void *c_rope, const void *win, const float *sinks, int32_t B,
                          int32_t H, int32_t D, int64_t T, int32_t HI, int32_t dI, int32_t k, int32_t W,
                          int32_t rope_dim, int64_t P, double theta_tok, double theta_cmp, float softmax_scale,
                          int32_t *idx_out, float *o, void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_CHECK_ARG(B >= 0 && H > 0 && D > 0 && T >= 0 && HI > 0 && dI > 0 && k >= 1 && W >= 0 && P >= 0);
    CSA_CHECK_ARG(decode_sizes_representable(B, T, k));
    CSA_CHECK_ARG(rope_dim >= 0 && rope_dim <= D && (rope_dim % 2) == 0);
    CSA_CHECK_ARG(rope_dim == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_ARG(B == 0 || (q != nullptr && qI_codes != nullptr && qI_scales != nullptr && w != nullptr &&
                             sinks != nullptr && o != nullptr));
    CSA_CHECK_ARG(B == 0 || T == 0 || (kI_codes != nullptr && kI_scales != nullptr));
    CSA_CHECK_ARG(B == 0 || W == 0 || win != nullptr);
    const bool fp8 = C == nullptr;
    CSA_CHECK_ARG(B == 0 || T == 0 || !fp8 || (c8 != nullptr && c8_scale != nullptr && c_rope != nullptr));
    CSA_CHECK_SUP(D == 64 || D == 128 || D == 256 || D == 512);
    CSA_CHECK_SUP(rope_dim % 8 == 0 && k <= 4096);
    CSA_CHECK_SUP((dI == 64 || dI == 128) && (HI == 16 || HI == 32 || HI == 64 || HI == 128));
    CSA_CHECK_SUP(T == 0 || decode_index_fp4_supported(T, HI, dI, k));
    CSA_CHECK_ARG(aligned16(q) && aligned16(qI_codes) && aligned16(kI_codes) && aligned16(C) && aligned16(c8) &&
                  aligned16(c_rope) && aligned16(win) && aligned16(o));
    CSA_TRY(check_workspace(workspace, workspace_bytes, decode_workspace_min(B, T, k)));
    cudaStream_t st = as_stream(stream);
    char *base = static_cast<char *>(workspace);
    float *scores = reinterpret_cast<float *>(base + kStatusBytes);
    const size_t index_ws = decode_index_bytes(B, T, k);
    int32_t *idx = idx_out != nullptr ? idx_out : reinterpret_cast<int32_t *>(base + kStatusBytes + index_ws);
    if (T > 0) {
        CSA_CUDA(cudaMemsetAsync(workspace, 0, kStatusBytes + decode_index_head_bytes(B), st));
        CSA_CUDA(launch_decode_index_fp4(qI_codes, qI_scales, w, kI_codes, kI_scales, B, T, HI, dI, k, idx, scores,
                                         static_cast<int32_t *>(workspace), st));
    } else {   // no entries: every index slot is -1
        CSA_TRY(reset_status(workspace, st));
        CSA_CUDA(launch_topk_rows(scores, B, 0, 0, 1, 1, k, idx, st));
    }
    return decode_attention(q, C, c8, c8_scale, c_rope, win, sinks, B, H, D, T, k, W, rope_dim, P, theta_tok, theta_cmp,
                            softmax_scale, idx, o, workspace, workspace_bytes, st);
}

csa_status hca_decode(const void *q, const void *C, const uint8_t *c8, const float *c8_scale, const void *c_rope,
                      const void *win, const float *sinks, int32_t B, int32_t H, int32_t D, int64_t T, int32_t W,
                      int32_t rope_dim, int64_t P, double theta_tok, double theta_cmp, float softmax_scale, float *o,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    CSA_CHECK_ARG(B >= 0 && H > 0 && D > 0 && T >= 0 && W >= 0 && P >= 0);
    CSA_CHECK_ARG(rope_dim >= 0 && rope_dim <= D && (rope_dim % 2) == 0);
    CSA_CHECK_ARG(rope_dim == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_ARG(B == 0 || (q != nullptr && sinks != nullptr && o != nullptr));
    CSA_CHECK_ARG(B == 0 || W == 0 || win != nullptr);
    const bool fp8 = C == nullptr;
    CSA_CHECK_ARG(B == 0 || T == 0 || !fp8 || (c8 != nullptr && c8_scale != nullptr && c_rope != nullptr));
    CSA_CHECK_SUP(D == 64 || D == 128 || D == 256 || D == 512);
    CSA_CHECK_SUP(rope_dim % 8 == 0);
    CSA_CHECK_ARG(aligned16(q) && aligned16(C) && aligned16(c8) && aligned16(c_rope) && aligned16(win) && aligned16(o));
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    AttnArgs a;
    memset(&a, 0, sizeof a);
    a.q = static_cast<const uint16_t *>(q);
    a.win = static_cast<const uint16_t *>(win);
    a.C = static_cast<const uint16_t *>(C);
    a.c8 = c8;
    a.c8_scale = c8_scale;
    a.c_rope = static_cast<const uint16_t *>(c_rope);
    a.idx = nullptr;   // every cached entry
    a.sinks = sinks;
    a.o = o;
    a.status = static_cast<int32_t *>(workspace);
    a.R = B;
    a.T = T;
    a.P = P;
    a.H = H;
    a.D = D;
    a.k = 0;
    a.W = W;
    a.r = rope_dim;
    a.m = 1;
    a.decode = 1;
    a.scale = softmax_scale > 0.f ? softmax_scale : (float)(1.0 / sqrt((double)D));
    a.log2_theta_tok = rope_dim > 0 ? log2(theta_tok) : 0.0;
    a.log2_theta_cmp = rope_dim > 0 ? log2(theta_cmp) : 0.0;
    if (attend_tc_supported(H, D, rope_dim, 0)) {
        int nsplit = hca_decode_splits_preferred(B, T, W);
        while (nsplit > 1 && kStatusBytes + align256(attend_tc_decode_partials(B, nsplit)) > workspace_bytes) --nsplit;
        return from_cuda(launch_attend_tc_decode(a, nsplit,
                                                 reinterpret_cast<float *>(static_cast<char *>(workspace) + kStatusBytes), st));
    }
    return from_cuda(launch_attend_simt(a, st));
}

csa_status swa_attend(const void *q, const void *kv_rot, const float *sinks, int64_t S, int64_t pos0, int32_t H,
                      int32_t D, int32_t W, int32_t rope_dim, double theta_tok, float softmax_scale, float *o,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    // the HCA attention with no compressed entries (both rope branches at theta_tok)
    return hca_attend(q, nullptr, kv_rot, sinks, S, pos0, H, D, 0, W, rope_dim, 1, theta_tok, theta_tok, softmax_scale,
                      o, workspace, workspace_bytes, stream);
}

csa_status csa_compress_append(const void *x_new, const void *g_new, const float *pos_bias, void *state_x,
                               void *state_g, int32_t B, int32_t D, int32_t m, int32_t L, int32_t rope_dim, int64_t P,
                               double theta_cmp, double theta_tok, void *C, uint8_t *c8, float *c8_scale, void *c_rope,
                               int64_t Tcap, void *win, int32_t W, void *stream)
{
    CSA_CHECK_ARG(B >= 0 && D > 0 && m >= 1 && L >= m && P >= 0 && Tcap >= 0 && W >= 0);
    CSA_CHECK_ARG(rope_dim >= 0 && rope_dim <= D && (rope_dim % 2) == 0);
    CSA_CHECK_ARG(rope_dim == 0 || (theta_ok(theta_cmp) && theta_ok(theta_tok)));
    CSA_CHECK_SUP(D % 8 == 0 && D <= 512 && rope_dim % 8 == 0);
    CSA_CHECK_ARG(B == 0 || (x_new != nullptr && g_new != nullptr && pos_bias != nullptr && state_x != nullptr &&
                             state_g != nullptr));
    CSA_CHECK_ARG(W == 0 || B == 0 || win != nullptr);
    const bool emits = (P + 1) % m == 0;
    const bool fp8 = C == nullptr;
    // an entry closing at P must fit the caller's cache, in one of the two formats
    CSA_CHECK_ARG(!emits || B == 0 || ((P + 1) / m - 1 < Tcap &&
                                       (!fp8 || (c8 != nullptr && c8_scale != nullptr &&
                                                 (rope_dim == 0 || c_rope != nullptr)))));
    CSA_CHECK_ARG(aligned16(x_new) && aligned16(g_new) && aligned16(state_x) && aligned16(state_g) && aligned16(C) &&
                  aligned16(c_rope) && aligned16(win));
    CSA_CHECK_ARG(fp8 == false || c8 == nullptr || ((reinterpret_cast<uintptr_t>(c8) & 7u) == 0 && (D - rope_dim) % 8 == 0));
    AppendArgs a;
    memset(&a, 0, sizeof a);
    a.x_new = static_cast<const uint16_t *>(x_new);
    a.g_new = static_cast<const uint16_t *>(g_new);
    a.bias = pos_bias;
    a.state_x = static_cast<uint16_t *>(state_x);
    a.state_g = static_cast<uint16_t *>(state_g);
    a.C = static_cast<uint16_t *>(C);
    a.c8 = c8;
    a.c8_scale = c8_scale;
    a.c_rope = static_cast<uint16_t *>(c_rope);
    a.win = W > 0 ? static_cast<uint16_t *>(win) : nullptr;
    a.P = P;
    a.Tcap = Tcap;
    a.B = B;
    a.D = D;
    a.m = m;
    a.L = L;
    a.r = rope_dim;
    a.W = W;
    a.log2_theta_cmp = rope_dim > 0 ? log2(theta_cmp) : 0.0;
    a.log2_theta_tok = rope_dim > 0 ? log2(theta_tok) : 0.0;
    return from_cuda(launch_compress_append(a, as_stream(stream)));
}

csa_status csa_out_proj(const void *o, const void *wa, const void *wb, int64_t S, int32_t H, int32_t D, int32_t G,
                        int32_t R, int32_t hidden, void *z, void *out, void *workspace, size_t workspace_bytes,
                        void *stream)
{
    CSA_CHECK_ARG(S >= 0 && H > 0 && D > 0 && G > 0 && R > 0 && hidden > 0 && H % G == 0);
    CSA_CHECK_ARG(S == 0 || (o != nullptr && wa != nullptr && wb != nullptr && z != nullptr && out != nullptr));
    CSA_CHECK_ARG(aligned16(o) && aligned16(wa) && aligned16(wb) && aligned16(z) && aligned16(out));
    const int64_t K = (int64_t)(H / G) * D;
    CSA_CHECK_SUP(K <= (1 << 30) && (int64_t)G * R <= (1 << 30));
    CSA_CHECK_SUP(csa::proj_gemm_tc_supported(std::max<int64_t>(S, 1), R, (int)K, G) &&
                  csa::proj_gemm_tc_supported(std::max<int64_t>(S, 1), hidden, G * R, 1));
    CSA_TRY(check_workspace(workspace, workspace_bytes, kStatusBytes));
    cudaStream_t st = as_stream(stream);
    CSA_TRY(reset_status(workspace, st));
    int32_t *status = static_cast<int32_t *>(workspace);
    CSA_CUDA(csa::launch_proj_gemm_tc(static_cast<const uint16_t *>(o), (int64_t)H * D, static_cast<const uint16_t *>(wa),
                                      static_cast<uint16_t *>(z), (int64_t)G * R, S, R, (int)K, G, status, st));
    return from_cuda(csa::launch_proj_gemm_tc(static_cast<const uint16_t *>(z), (int64_t)G * R,
                                              static_cast<const uint16_t *>(wb), static_cast<uint16_t *>(out), hidden, S,
                                              hidden, G * R, 1, status, st));
}

}  // extern "C"
