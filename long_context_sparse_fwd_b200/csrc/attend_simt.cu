// attend_simt.cu -- shared-K=V multi-query attention over (window rows + compressed entries) with
// a per-head sink: the general CUDA-core path. It serves every shape the tensor-core kernels do
// not take (small heads/dims, decode) and is the GPU-side cross-check for them.
//
// Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention": one KV head read as
// both key and value; partial interleaved RoPE on the last qk_rope_head_dim channels, with the
// output rope slice rotated at position -i (eq. 26) so each key contributes as a function of its
// distance to the query; a learnable per-head sink (eq. 27) in the softmax denominator; the
// compressed entries are concatenated with a sliding window of raw K=V rows. Section "Attention
// mask layout": the window covers keys (i - window, i]; CSA keys are the indexer's picks (-1 =
// empty slot); HCA keys are every entry w < (i+1)//m.
//
// Window rows are rotated with theta_tok and entries with theta_cmp (llm-atlas "DeepSeek-V4-Flash"
// config: rope_theta / compress_rope_theta), so q is rotated once per branch and each branch's
// rope slice is rotated back with its own theta.
//
// Layout: one CTA per (query row, group of 8 heads), one warp per head. Keys stream through
// shared memory in tiles of 32 (each lane scores one key against the broadcast query, then the
// tile's probabilities are broadcast for the value pass). The sink seeds the running max / sum,
// so it is counted exactly once.
#include <cuda_fp8.h>

#include "kernels.cuh"

namespace csa {


constexpr int HG = 8;         // heads per CTA (one warp each)
constexpr int KT = 32;        // keys per tile

template <int NI>  // NI = D / 32 values per lane
__global__ void __launch_bounds__(256, 2)
attend_simt_kernel(AttnArgs a)
{
    constexpr int D = NI * 32;
    extern __shared__ float smem[];
    float *qt = smem;                      // [HG][D] query rotated with theta_tok
    float *qc = qt + HG * D;               // [HG][D] query rotated with theta_cmp
    float *ks = qc + HG * D;               // [KT][D+1] key tile
    int *elist = reinterpret_cast<int *>(ks + KT * (D + 1));   // compacted entry list [k]

    const int64_t row = blockIdx.x;
    const int h0 = blockIdx.y * HG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = h0 + warp;
    const int64_t t = a.decode ? a.P : a.pos0 + row;
    const int r = a.r;

    // ---- rotated query copies ----
    for (int i = threadIdx.x; i < HG * (D / 2); i += blockDim.x) {
        const int hh = i / (D / 2), pr = i % (D / 2);
        const int d = 2 * pr;
        float x0 = 0.f, x1 = 0.f;
        if (h0 + hh < a.H) {
            const uint32_t v = *reinterpret_cast<const uint32_t *>(a.q + ((row * a.H) + h0 + hh) * (int64_t)D + d);
            x0 = bf_lo(v); x1 = bf_hi(v);
        }
        if (d >= D - r) {
            const int p = (d - (D - r)) >> 1;
            float c, s;
            rope_cos_sin((double)t, p, r, a.log2_theta_tok, &c, &s);
            qt[hh * D + d] = x0 * c - x1 * s;
            qt[hh * D + d + 1] = x0 * s + x1 * c;
            rope_cos_sin((double)t, p, r, a.log2_theta_cmp, &c, &s);
            qc[hh * D + d] = x0 * c - x1 * s;
            qc[hh * D + d + 1] = x0 * s + x1 * c;
        } else {
            qt[hh * D + d] = x0; qt[hh * D + d + 1] = x1;
            qc[hh * D + d] = x0; qc[hh * D + d + 1] = x1;
        }
    }

    // ---- key lists ----
    const int64_t vis = a.decode ? a.T : visible_entries(t, a.m, a.T);
    int nw = 0;               // window rows: positions t-W+1 .. t that are >= 0
    int64_t wpos0 = t - a.W + 1;
    if (wpos0 < 0) wpos0 = 0;
    nw = (int)(t - wpos0 + 1);
    if (a.W == 0) nw = 0;
    int ne = 0;
    if (a.idx != nullptr) {
        if (warp == 0) {
            const int32_t *ir = a.idx + row * (int64_t)a.k;
            int cnt = 0;
            for (int base = 0; base < a.k; base += 32) {
                const int j = base + lane;
                int s = j < a.k ? ir[j] : -1;
                bool ok = s >= 0 && (int64_t)s < vis;
                if (s >= 0 && !ok) report(a.status, CSA_ERR_INVALID_ARG);
                const unsigned mk = __ballot_sync(0xffffffffu, ok);
                if (ok) elist[cnt + __popc(mk & ((1u << lane) - 1u))] = s;
                cnt += __popc(mk);
            }
            if (lane == 0) elist[a.k] = cnt;
        }
        __syncthreads();
        ne = elist[a.k];
    } else {
        ne = (int)vis;
        __syncthreads();
    }

    const bool active = h < a.H;
    const float z = active ? a.sinks[h] : 0.f;
    float m_run = z, l_run = 1.f;     // the sink seeds the softmax state: exp(z - z) = 1, no value
    float accw[NI], acce[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) { accw[i] = 0.f; acce[i] = 0.f; }

    const int ntiles_w = (nw + KT - 1) / KT;
    const int ntiles_e = (ne + KT - 1) / KT;
    for (int tile = 0; tile < ntiles_w + ntiles_e; ++tile) {
        const bool is_win = tile < ntiles_w;
        const int kbase = is_win ? tile * KT : (tile - ntiles_w) * KT;
        const int nk = min(KT, (is_win ? nw : ne) - kbase);
        __syncthreads();
        // load the tile (bf16 / fp8 -> fp32 in shared memory)
        for (int i = threadIdx.x; i < nk * (D / 8); i += blockDim.x) {
            const int j = i / (D / 8), c0 = (i % (D / 8)) * 8;
            float v[8];
            if (is_win) {
                const uint16_t *src = a.decode
                    ? a.win + (row * a.W + (a.W - nw) + kbase + j) * (int64_t)D
                    : a.win + (wpos0 + kbase + j) * (int64_t)D;
                const uint4 u = *reinterpret_cast<const uint4 *>(src + c0);
                const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) { v[2 * e] = bf_lo(uw[e]); v[2 * e + 1] = bf_hi(uw[e]); }
            } else {
                const int64_t s = a.idx != nullptr ? (int64_t)elist[kbase + j] : (int64_t)(kbase + j);
                const int64_t erow = (a.decode ? row * a.T : 0) + s;
                if (a.C != nullptr) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(a.C + erow * D + c0);
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) { v[2 * e] = bf_lo(uw[e]); v[2 * e + 1] = bf_hi(uw[e]); }
                } else if (c0 < D - r) {
                    const float sc = a.c8_scale[erow];
                    const uint2 u = *reinterpret_cast<const uint2 *>(a.c8 + erow * (int64_t)(D - r) + c0);
                    const uint32_t uw[2] = {u.x, u.y};
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const __nv_fp8_e4m3 f = *reinterpret_cast<const __nv_fp8_e4m3 *>(
                            reinterpret_cast<const uint8_t *>(uw) + e);
                        v[e] = float(f) * sc;
                    }
                } else {
                    const uint4 u = *reinterpret_cast<const uint4 *>(a.c_rope + erow * (int64_t)r + (c0 - (D - r)));
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) { v[2 * e] = bf_lo(uw[e]); v[2 * e + 1] = bf_hi(uw[e]); }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) ks[j * (D + 1) + c0 + e] = v[e];
        }
        __syncthreads();
        if (!active) continue;
        // logits: lane j scores key j
        const float *qv = (is_win ? qt : qc) + warp * D;
        float logit = -INFINITY;
        if (lane < nk) {
            const float *kr = ks + lane * (D + 1);
            float dot = 0.f;
#pragma unroll 8
            for (int d = 0; d < D; ++d) dot = fmaf(qv[d], kr[d], dot);
            logit = dot * a.scale;
        }
        float tmax = logit;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
        const float m_new = fmaxf(m_run, tmax);
        const float corr = expf(m_run - m_new);
        const float p = lane < nk ? expf(logit - m_new) : 0.f;
        float psum = p;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
        l_run = l_run * corr + psum;
        m_run = m_new;
#pragma unroll
        for (int i = 0; i < NI; ++i) { accw[i] *= corr; acce[i] *= corr; }
        for (int j = 0; j < nk; ++j) {
            const float pj = __shfl_sync(0xffffffffu, p, j);
            const float *kr = ks + j * (D + 1);
            if (is_win) {
#pragma unroll
                for (int i = 0; i < NI; ++i) accw[i] = fmaf(pj, kr[lane + 32 * i], accw[i]);
            } else {
#pragma unroll
                for (int i = 0; i < NI; ++i) acce[i] = fmaf(pj, kr[lane + 32 * i], acce[i]);
            }
        }
    }
    if (!active) return;
    // ---- rotate each branch's rope slice back by -t, normalise, store ----
    const float inv_l = 1.f / l_run;
    float *orow = a.o + ((row * a.H) + h) * (int64_t)D;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        const int d = lane + 32 * i;
        float vw = accw[i], ve = acce[i];
        const float pw = __shfl_xor_sync(0xffffffffu, vw, 1);
        const float pe = __shfl_xor_sync(0xffffffffu, ve, 1);
        if (d >= D - r) {
            const int p = (d - (D - r)) >> 1;
            float c, s;
            // rotation by -t: (x, y) -> (x c + y s, -x s + y c)
            rope_cos_sin((double)t, p, r, a.log2_theta_tok, &c, &s);
            vw = (lane & 1) ? (-pw * s + vw * c) : (vw * c + pw * s);
            rope_cos_sin((double)t, p, r, a.log2_theta_cmp, &c, &s);
            ve = (lane & 1) ? (-pe * s + ve * c) : (ve * c + pe * s);
        }
        orow[d] = (vw + ve) * inv_l;
    }
}

size_t attend_simt_smem(int D, int k)
{
    return sizeof(float) * (size_t)(2 * HG * D + KT * (D + 1)) + sizeof(int) * (size_t)(k + 1);
}

cudaError_t launch_attend_simt(const AttnArgs &a, cudaStream_t stream)
{
    if (a.R == 0) return cudaSuccess;
    dim3 grid((unsigned)a.R, (unsigned)((a.H + HG - 1) / HG));
    const size_t smem = attend_simt_smem(a.D, a.k);
    switch (a.D) {
#define CSA_CASE(NIV)                                                                                         \
    case NIV * 32:                                                                                            \
        cudaFuncSetAttribute(attend_simt_kernel<NIV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        attend_simt_kernel<NIV><<<grid, 256, smem, stream>>>(a);                                              \
        break;
        CSA_CASE(2)
        CSA_CASE(4)
        CSA_CASE(8)
        CSA_CASE(16)
#undef CSA_CASE
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace csa
