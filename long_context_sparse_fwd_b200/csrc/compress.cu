// compress.cu -- softmax-gated KV compressor (CSA m=4 / window 2m; HCA m'=128 / window m') and
// the RoPE'd raw-row copy for the sliding-window branch.
//
// Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention": CSA pools every m
// tokens into one entry over overlapping windows, HCA over non-overlapping windows of m'; the
// insight.ai.kr digest of the HF blog: the pooling is a softmax gate with a learned position
// bias. Entry w pools [(w+1)m - L, (w+1)m) clipped to [0,S); per channel the weights are a
// softmax over positions of gate + bias[offset]; the entry is rotated at position w*m with
// compress_rope_theta (llm-atlas "DeepSeek-V4-Flash", config.json table).
//
// HBM-bound streaming: each thread owns 8 channels (one 16-byte vector) of one entry and walks
// the window with an online softmax in fp32; overlapping CSA windows re-read the previous block
// from L2. The raw-row kernel reads each kv row once and writes it rotated at its own position.
#include "kernels.cuh"

namespace csa {

__global__ void __launch_bounds__(256)
compress_entries_kernel(const uint16_t *__restrict__ kv, const uint16_t *__restrict__ gate,
                        const float *__restrict__ bias, int64_t T, int D, int m, int L, int r,
                        double log2_theta_cmp, uint16_t *__restrict__ C)
{
    const int chunks = D >> 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= T * chunks) return;
    const int64_t w = gid / chunks;
    const int d0 = (int)(gid - w * chunks) << 3;
    const int64_t start = (w + 1) * (int64_t)m - L;
    const int64_t end = (w + 1) * (int64_t)m;
    const int64_t lo = start < 0 ? 0 : start;

    float mx[8], l[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; l[e] = 0.f; acc[e] = 0.f; }

#pragma unroll 4
    for (int64_t j = lo; j < end; ++j) {
        const uint4 g = __ldg(reinterpret_cast<const uint4 *>(gate + j * D + d0));
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(kv + j * D + d0));
        const float b = __ldg(bias + (j - start));
        const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float a = ((e & 1) ? bf_hi(gw[e >> 1]) : bf_lo(gw[e >> 1])) + b;
            const float x = (e & 1) ? bf_hi(vw[e >> 1]) : bf_lo(vw[e >> 1]);
            if (a > mx[e]) {
                const float corr = expf(mx[e] - a);
                l[e] = l[e] * corr + 1.f;
                acc[e] = acc[e] * corr + x;
                mx[e] = a;
            } else {
                const float p = expf(a - mx[e]);
                l[e] += p;
                acc[e] += p * x;
            }
        }
    }
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = acc[e] / l[e];
    if (d0 >= D - r) {
        const double pos = (double)(w * (int64_t)m);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const int p = (d0 + e - (D - r)) >> 1;
            float c, s;
            rope_cos_sin(pos, p, r, log2_theta_cmp, &c, &s);
            const float x0 = out[e], x1 = out[e + 1];
            out[e] = x0 * c - x1 * s;
            out[e + 1] = x0 * s + x1 * c;
        }
    }
    uint4 o;
    o.x = pack_bf2(out[0], out[1]);
    o.y = pack_bf2(out[2], out[3]);
    o.z = pack_bf2(out[4], out[5]);
    o.w = pack_bf2(out[6], out[7]);
    *reinterpret_cast<uint4 *>(C + w * D + d0) = o;
}

// Long windows (HCA: L = 128): the window of one (entry, 8-channel group) is split across G = 8
// neighbouring lanes, each walking L/G consecutive positions with its own online softmax; the G
// partial (max, sum, weighted sum) states are then merged by shuffles. Lane j of a group of 8 lanes
// takes positions j*L/8 ..; the 4 groups of a warp take 4 consecutive channel groups (64 contiguous
// bytes of each row).
__global__ void __launch_bounds__(256)
compress_entries_split_kernel(const uint16_t *__restrict__ kv, const uint16_t *__restrict__ gate,
                              const float *__restrict__ bias, int64_t T, int D, int m, int L, int r,
                              double log2_theta_cmp, uint16_t *__restrict__ C)
{
    constexpr int G = 8;
    const int chunks = D >> 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int sub = threadIdx.x & (G - 1);
    const int64_t item = gid / G;   // (entry, channel group)
    const bool valid = item < T * chunks;
    const int64_t w = valid ? item / chunks : 0;
    const int d0 = valid ? (int)(item - w * chunks) << 3 : 0;
    const int64_t start = (w + 1) * (int64_t)m - L;
    const int64_t end = (w + 1) * (int64_t)m;
    const int per = (L + G - 1) / G;
    int64_t j0 = start + (int64_t)sub * per, j1 = j0 + per;
    if (j0 < 0) j0 = 0;
    if (j1 > end) j1 = end;

    float mx[8], l[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; l[e] = 0.f; acc[e] = 0.f; }
    if (valid) {
#pragma unroll 4
        for (int64_t j = j0; j < j1; ++j) {
            const uint4 g = __ldg(reinterpret_cast<const uint4 *>(gate + j * D + d0));
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(kv + j * D + d0));
            const float b = __ldg(bias + (j - start));
            const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
            const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float a = ((e & 1) ? bf_hi(gw[e >> 1]) : bf_lo(gw[e >> 1])) + b;
                const float x = (e & 1) ? bf_hi(vw[e >> 1]) : bf_lo(vw[e >> 1]);
                if (a > mx[e]) {
                    const float corr = expf(mx[e] - a);
                    l[e] = l[e] * corr + 1.f;
                    acc[e] = acc[e] * corr + x;
                    mx[e] = a;
                } else {
                    const float pe = expf(a - mx[e]);
                    l[e] += pe;
                    acc[e] += pe * x;
                }
            }
        }
    }
    // merge the G partial states of this (entry, channel group): lanes differing in the low 3 bits
#pragma unroll
    for (int o = 1; o < G; o <<= 1) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float m2 = __shfl_xor_sync(0xffffffffu, mx[e], o);
            const float l2 = __shfl_xor_sync(0xffffffffu, l[e], o);
            const float a2 = __shfl_xor_sync(0xffffffffu, acc[e], o);
            const float mm = fmaxf(mx[e], m2);
            const float c1 = mx[e] == -INFINITY ? 0.f : expf(mx[e] - mm);
            const float c2 = m2 == -INFINITY ? 0.f : expf(m2 - mm);
            l[e] = l[e] * c1 + l2 * c2;
            acc[e] = acc[e] * c1 + a2 * c2;
            mx[e] = mm;
        }
    }
    if (!valid || sub != 0) return;
    float out[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) out[e] = acc[e] / l[e];
    if (d0 >= D - r) {
        const double pos = (double)(w * (int64_t)m);
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            const int pp = (d0 + e - (D - r)) >> 1;
            float c, sn;
            rope_cos_sin(pos, pp, r, log2_theta_cmp, &c, &sn);
            const float x0 = out[e], x1 = out[e + 1];
            out[e] = x0 * c - x1 * sn;
            out[e + 1] = x0 * sn + x1 * c;
        }
    }
    uint4 o4;
    o4.x = pack_bf2(out[0], out[1]);
    o4.y = pack_bf2(out[2], out[3]);
    o4.z = pack_bf2(out[4], out[5]);
    o4.w = pack_bf2(out[6], out[7]);
    *reinterpret_cast<uint4 *>(C + w * D + d0) = o4;
}

__global__ void __launch_bounds__(256)
rotate_rows_kernel(const uint16_t *__restrict__ kv, int64_t S, int D, int r, double log2_theta_tok,
                   uint16_t *__restrict__ kv_rot)
{
    const int chunks = D >> 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= S * chunks) return;
    const int64_t j = gid / chunks;
    const int d0 = (int)(gid - j * chunks) << 3;
    uint4 v = __ldg(reinterpret_cast<const uint4 *>(kv + j * D + d0));
    if (d0 >= D - r) {
        uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int p = (d0 + 2 * e - (D - r)) >> 1;
            float c, s;
            rope_cos_sin((double)j, p, r, log2_theta_tok, &c, &s);
            const float x0 = bf_lo(vw[e]), x1 = bf_hi(vw[e]);
            vw[e] = pack_bf2(x0 * c - x1 * s, x0 * s + x1 * c);
        }
        v.x = vw[0]; v.y = vw[1]; v.z = vw[2]; v.w = vw[3];
    }
    *reinterpret_cast<uint4 *>(kv_rot + j * D + d0) = v;
}

cudaError_t launch_compress(const uint16_t *kv, const uint16_t *gate, const float *bias, int64_t S, int D,
                            int m, int L, int r, double theta_cmp, double theta_tok, uint16_t *C,
                            uint16_t *kv_rot, cudaStream_t stream)
{
    const int64_t T = S / m;
    const int chunks = D / 8;
    if (T > 0 && C != nullptr) {
        const int64_t n = T * chunks;
        if (L >= 64) {   // long windows: split each window across 8 lanes
            const int64_t nt = n * 8;
            compress_entries_split_kernel<<<(unsigned)((nt + 255) / 256), 256, 0, stream>>>(kv, gate, bias, T, D, m, L,
                                                                                             r, log2(theta_cmp), C);
        } else {
            compress_entries_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(kv, gate, bias, T, D, m, L, r,
                                                                                      log2(theta_cmp), C);
        }
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (S > 0 && kv_rot != nullptr) {
        const int64_t n = S * chunks;
        rotate_rows_kernel<<<(unsigned)((n + 255) / 256), 256, 0, stream>>>(kv, S, D, r, log2(theta_tok), kv_rot);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

}  // namespace csa
