// index_topk.cu -- lightning-indexer scores and exact top-k selection (general path).
//
// Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention" (CSA): a lightning
// indexer scores each query against the compressed pool and keeps the top index_topk entries;
// insight.ai.kr digest of the HF blog: the score is a ReLU multi-head dot product. Here
// I[r,s] = sum_h w[r,h] * ReLU(qI[r,h,:] . kI[s,:]) for visible s ("Attention mask layout":
// entry w is visible to query t iff w < (t+1)//m; unfilled slots carry -1).
//
// Selection is exact: the fp32 score is mapped to an order-preserving uint32 key, a 4-pass
// 8-bit radix select finds the k-th largest key, then one ordered block scan keeps every key
// above it plus the lowest-index keys equal to it (ties go to the smaller entry index). The
// kept indices are written in ascending order, so the result does not depend on launch shape.
#include "kernels.cuh"

namespace csa {

// ---- scores: one CTA per (row, 256 entries); grid.x = rows, grid.y = entry chunks; q row staged in shared memory as fp32 ----------------
template <int DI>
__global__ void __launch_bounds__(256)
index_scores_kernel(const uint16_t *__restrict__ qI, const float *__restrict__ w, const uint16_t *__restrict__ kI,
                    int64_t pos0, int64_t T, int HI, int m, int decode, float *__restrict__ scores)
{
    extern __shared__ float smem[];
    float *qs = smem;              // [HI][DI]
    float *ws = smem + HI * DI;    // [HI]
    const int64_t row = blockIdx.x;
    const int64_t vis = decode ? T : visible_entries(pos0 + row, m, T);
    const int64_t s0 = (int64_t)blockIdx.y * 256;
    if (s0 >= vis) return;
    const uint16_t *qrow = qI + row * (int64_t)HI * DI;
    for (int i = threadIdx.x; i < HI * DI; i += blockDim.x) qs[i] = bf2f(qrow[i]);
    for (int i = threadIdx.x; i < HI; i += blockDim.x) ws[i] = w[row * HI + i];
    __syncthreads();
    const int64_t s = s0 + threadIdx.x;
    if (s >= vis) return;
    const uint16_t *krow = kI + ((decode ? row * T : 0) + s) * DI;
    uint32_t kreg[DI / 2];
#pragma unroll
    for (int c = 0; c < DI / 8; ++c) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(krow) + c);
        kreg[4 * c + 0] = v.x; kreg[4 * c + 1] = v.y; kreg[4 * c + 2] = v.z; kreg[4 * c + 3] = v.w;
    }
    float total = 0.f;
    for (int h = 0; h < HI; ++h) {
        const float4 *qh = reinterpret_cast<const float4 *>(qs + h * DI);
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < DI / 4; ++c) {
            const float4 qv = qh[c];
            dot = fmaf(qv.x, bf_lo(kreg[2 * c]), dot);
            dot = fmaf(qv.y, bf_hi(kreg[2 * c]), dot);
            dot = fmaf(qv.z, bf_lo(kreg[2 * c + 1]), dot);
            dot = fmaf(qv.w, bf_hi(kreg[2 * c + 1]), dot);
        }
        total = fmaf(ws[h], fmaxf(dot, 0.f), total);
    }
    scores[row * T + s] = total + 0.0f;
}

// ---- exact top-k over one row of scores ---------------------------------------------------------------
constexpr int TOPK_THREADS = 1024;

// inclusive block scan of one int per thread; returns the inclusive prefix, *total = block sum
__device__ __forceinline__ int block_scan_incl(int v, int *warp_sums, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) warp_sums[wid] = v;
    __syncthreads();
    if (wid == 0) {
        const int nw = blockDim.x >> 5;
        int x = lane < nw ? warp_sums[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        if (lane < nw) warp_sums[lane] = x;
    }
    __syncthreads();
    const int before = wid > 0 ? warp_sums[wid - 1] : 0;
    *total = warp_sums[(blockDim.x >> 5) - 1];
    __syncthreads();
    return v + before;
}

__global__ void __launch_bounds__(TOPK_THREADS)
topk_rows_kernel(const float *__restrict__ scores, int64_t pos0, int64_t T, int m, int decode, int k,
                 int32_t *__restrict__ idx)
{
    __shared__ uint32_t hist[256];
    __shared__ int warp_sums[32];
    __shared__ uint32_t sh_prefix, sh_remaining;
    const int64_t row = blockIdx.x;
    const int64_t n = decode ? T : visible_entries(pos0 + row, m, T);
    const float *sc = scores + row * T;
    int32_t *out = idx + row * (int64_t)k;

    if (n <= k) {  // everything visible is selected
        for (int64_t i = threadIdx.x; i < k; i += blockDim.x) out[i] = i < n ? (int32_t)i : -1;
        return;
    }
    // radix select of the k-th largest key, 8 bits per pass from the top
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = score_key(sc[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (threadIdx.x == 0) {
            uint32_t cum = 0;
            int d = 255;
            for (; d > 0; --d) {
                if (cum + hist[d] >= remaining) break;
                cum += hist[d];
            }
            sh_prefix = prefix | ((uint32_t)d << shift);
            sh_remaining = remaining - cum;
        }
        __syncthreads();
        prefix = sh_prefix;
        remaining = sh_remaining;
        mask |= 255u << shift;
        __syncthreads();
    }
    // keep keys > prefix, and the first `remaining` keys == prefix in index order
    int eq_seen = 0, written = 0;
    for (int64_t base = 0; base < n; base += blockDim.x) {
        const int64_t i = base + threadIdx.x;
        uint32_t key = 0;
        if (i < n) key = score_key(sc[i]);
        const int is_eq = (i < n && key == prefix) ? 1 : 0;
        int eq_tot;
        const int eq_incl = block_scan_incl(is_eq, warp_sums, &eq_tot);
        const int eq_rank = eq_seen + eq_incl - is_eq;
        const int sel = (i < n) && (key > prefix || (is_eq && eq_rank < (int)remaining)) ? 1 : 0;
        int sel_tot;
        const int sel_incl = block_scan_incl(sel, warp_sums, &sel_tot);
        if (sel) out[written + sel_incl - 1] = (int32_t)i;
        eq_seen += eq_tot;
        written += sel_tot;
        if (written >= k) break;   // uniform across the block
    }
}

cudaError_t launch_index_scores(const uint16_t *qI, const float *w, const uint16_t *kI, int64_t R, int64_t pos0,
                                int64_t T, int HI, int dI, int m, int decode, float *scores, cudaStream_t stream)
{
    if (R == 0 || T == 0) return cudaSuccess;
    dim3 grid((unsigned)R, (unsigned)((T + 255) / 256));
    const size_t smem = sizeof(float) * (size_t)(HI * dI + HI);
    switch (dI) {
#define CSA_CASE(DV)                                                                                  \
    case DV:                                                                                          \
        if (smem > 48 * 1024)                                                                         \
            cudaFuncSetAttribute(index_scores_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, \
                                 (int)smem);                                                          \
        index_scores_kernel<DV><<<grid, 256, smem, stream>>>(qI, w, kI, pos0, T, HI, m, decode, scores); \
        break;
        CSA_CASE(32)
        CSA_CASE(64)
        CSA_CASE(128)
        CSA_CASE(256)
#undef CSA_CASE
    default:
        return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_topk_rows(const float *scores, int64_t R, int64_t pos0, int64_t T, int m, int decode, int k,
                             int32_t *idx, cudaStream_t stream)
{
    if (R == 0) return cudaSuccess;
    topk_rows_kernel<<<(unsigned)R, TOPK_THREADS, 0, stream>>>(scores, pos0, T, m, decode, k, idx);
    return cudaGetLastError();
}

}  // namespace csa
