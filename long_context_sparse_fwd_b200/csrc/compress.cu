// compress.cu -- softmax-gated KV compressor (CSA m=4 / window 2m; HCA m'=128 / window m') fused with
// the RoPE'd raw-row copy for the sliding-window branch, for a prefill chunk at positions
// pos0 .. pos0+S-1 (pos0 = 0 for a whole prefill).
//
// Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention": CSA pools every m
// tokens into one entry over overlapping windows, HCA over non-overlapping windows of m'; the
// insight.ai.kr digest of the HF blog: the pooling is a softmax gate with a learned position
// bias; section "Cache layers": state carries over between forward calls. Entry w pools
// [(w+1)m - L, (w+1)m) clipped at position 0; per channel the weights are a softmax over positions of
// gate + bias[offset]; the entry is rotated at position w*m with compress_rope_theta (llm-atlas
// "DeepSeek-V4-Flash", config.json table). A chunk writes the entries whose window closes inside it,
// w in [floor(pos0/m), floor((pos0+S)/m)), and the window rows of its own positions.
//
// HBM-bound streaming, one launch with two roles: the first CTAs pool the entries (one thread per entry
// and 8-channel group walking the window with an online softmax in fp32, 16-byte vectors; these are
// the longer dependency chains, so they start first); the rest write the chunk's rows rotated at
// their own position with theta_tok (one thread per row and 8-channel group). Long windows (HCA,
// L >= 64) split each entry's window across 8 lanes whose online-softmax states are merged by shuffles.
#include "kernels.cuh"

namespace csa {

namespace {

// Row j of kv rotated at position j with theta_tok on the rope channels this 8-channel group holds.
__device__ __forceinline__ uint4 rotate_row8(uint4 v, int64_t j, int d0, int D, int r, double log2_theta_tok)
{
    if (d0 < D - r) return v;
    uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int p = (d0 + 2 * e - (D - r)) >> 1;
        float c, s;
        rope_cos_sin((double)j, p, r, log2_theta_tok, &c, &s);
        const float x0 = bf_lo(vw[e]), x1 = bf_hi(vw[e]);
        vw[e] = pack_bf2(x0 * c - x1 * s, x0 * s + x1 * c);
    }
    return make_uint4(vw[0], vw[1], vw[2], vw[3]);
}

// One online-softmax step over the 8 channels of a row: gate logits g (+ bias b), values v.
__device__ __forceinline__ void pool_step(uint4 g, uint4 v, float b, float (&mx)[8], float (&l)[8], float (&acc)[8])
{
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

// Normalise, rotate at the entry position w*m with theta_cmp and store entry w's 8 channels.
__device__ __forceinline__ void store_entry8(const float (&l)[8], const float (&acc)[8], int64_t w, int m, int d0, int D,
                                             int r, double log2_theta_cmp, uint16_t *C)
{
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
    uint4 o;
    o.x = pack_bf2(out[0], out[1]);
    o.y = pack_bf2(out[2], out[3]);
    o.z = pack_bf2(out[4], out[5]);
    o.w = pack_bf2(out[6], out[7]);
    *reinterpret_cast<uint4 *>(C + w * D + d0) = o;
}

struct CompressArgs {
    const uint16_t *kv, *gate;   // [pos0 + S, D] by absolute position
    const float *bias;           // [L]
    uint16_t *C;                 // [T1, D] (entries [T0, T1) written)
    uint16_t *kv_rot;            // [pos0 + S, D] (rows [pos0, pos0 + S) written) or null
    int64_t pos0, end;           // chunk positions [pos0, end)
    int64_t T0, T1;              // entries [T0, T1) close inside the chunk
    int64_t pool_blocks;         // CTAs of the pooling role (the rest of the grid rotates rows)
    int D, m, L, r;
    double log2_theta_cmp, log2_theta_tok;
};

// Row role: one thread per (row, 8-channel group) of the chunk writes the row rotated at its position.
__device__ __forceinline__ void rotate_role(const CompressArgs &a, int64_t gid)
{
    const int chunks = a.D >> 3;
    const int64_t j = a.pos0 + gid / chunks;
    if (j >= a.end) return;
    const int d0 = (int)(gid % chunks) << 3;
    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.kv + j * a.D + d0));
    *reinterpret_cast<uint4 *>(a.kv_rot + j * a.D + d0) = rotate_row8(v, j, d0, a.D, a.r, a.log2_theta_tok);
}

// Short windows (CSA, L = 2m): the row role, then one thread per (entry, 8-channel group) walking the
// entry's window with an online softmax.
__global__ void __launch_bounds__(256)
compress_fused_kernel(CompressArgs a)
{
    if (blockIdx.x >= a.pool_blocks) {
        rotate_role(a, (int64_t)(blockIdx.x - a.pool_blocks) * blockDim.x + threadIdx.x);
        return;
    }
    const int chunks = a.D >> 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t w = a.T0 + gid / chunks;
    if (w >= a.T1) return;
    const int d0 = (int)(gid % chunks) << 3;
    const int64_t start = (w + 1) * (int64_t)a.m - a.L, end = (w + 1) * (int64_t)a.m;
    float mx[8], l[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; l[e] = 0.f; acc[e] = 0.f; }
#pragma unroll 4
    for (int64_t j = start < 0 ? 0 : start; j < end; ++j) {
        const uint4 g = __ldg(reinterpret_cast<const uint4 *>(a.gate + j * a.D + d0));
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.kv + j * a.D + d0));
        pool_step(g, v, __ldg(a.bias + (j - start)), mx, l, acc);
    }
    store_entry8(l, acc, w, a.m, d0, a.D, a.r, a.log2_theta_cmp, a.C);
}

// Long windows (HCA: L = 128): the row role, then the window of one (entry, 8-channel group) split
// across G = 8 neighbouring lanes, each walking L/G consecutive positions with its own online softmax;
// the G partial (max, sum, weighted sum) states are merged by shuffles. Lane j of a group of 8 lanes
// takes positions j*L/8 ..; the 4 groups of a warp take 4 consecutive channel groups (64 contiguous
// bytes of each row).
__global__ void __launch_bounds__(256)
compress_fused_split_kernel(CompressArgs a)
{
    if (blockIdx.x >= a.pool_blocks) {
        rotate_role(a, (int64_t)(blockIdx.x - a.pool_blocks) * blockDim.x + threadIdx.x);
        return;
    }
    constexpr int G = 8;
    const int chunks = a.D >> 3;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int sub = threadIdx.x & (G - 1);
    const int64_t item = gid / G;   // (entry, channel group)
    const bool valid = item < (a.T1 - a.T0) * chunks;
    const int64_t w = a.T0 + (valid ? item / chunks : 0);
    const int d0 = valid ? (int)(item % chunks) << 3 : 0;
    const int64_t start = (w + 1) * (int64_t)a.m - a.L, end = (w + 1) * (int64_t)a.m;
    const int per = (a.L + G - 1) / G;
    int64_t j0 = start + (int64_t)sub * per, j1 = j0 + per;
    if (j0 < 0) j0 = 0;
    if (j1 > end) j1 = end;

    float mx[8], l[8], acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) { mx[e] = -INFINITY; l[e] = 0.f; acc[e] = 0.f; }
    if (valid) {
#pragma unroll 4
        for (int64_t j = j0; j < j1; ++j) {
            const uint4 g = __ldg(reinterpret_cast<const uint4 *>(a.gate + j * a.D + d0));
            const uint4 v = __ldg(reinterpret_cast<const uint4 *>(a.kv + j * a.D + d0));
            pool_step(g, v, __ldg(a.bias + (j - start)), mx, l, acc);
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
    store_entry8(l, acc, w, a.m, d0, a.D, a.r, a.log2_theta_cmp, a.C);
}

}  // namespace

cudaError_t launch_compress(const uint16_t *kv, const uint16_t *gate, const float *bias, int64_t S, int64_t pos0,
                            int D, int m, int L, int r, double theta_cmp, double theta_tok, uint16_t *C,
                            uint16_t *kv_rot, cudaStream_t stream)
{
    if (S <= 0) return cudaSuccess;
    CompressArgs a;
    a.kv = kv;
    a.gate = gate;
    a.bias = bias;
    a.C = C;
    a.kv_rot = kv_rot;
    a.pos0 = pos0;
    a.end = pos0 + S;
    a.T0 = pos0 / m;
    a.T1 = C != nullptr ? a.end / m : a.T0;   // no entry cache: rows only
    a.D = D;
    a.m = m;
    a.L = L;
    a.r = r;
    a.log2_theta_cmp = r > 0 ? log2(theta_cmp) : 0.0;
    a.log2_theta_tok = r > 0 ? log2(theta_tok) : 0.0;
    const int64_t chunks = D / 8;
    const int64_t items = (a.T1 - a.T0) * chunks * (L >= 64 ? 8 : 1);   // long windows: 8 lanes per item
    a.pool_blocks = (items + 255) / 256;                                 // the longer chains start first
    const int64_t grid = a.pool_blocks + (kv_rot != nullptr ? (S * chunks + 255) / 256 : 0);
    if (grid == 0) return cudaSuccess;
    if (L >= 64)
        compress_fused_split_kernel<<<(unsigned)grid, 256, 0, stream>>>(a);
    else
        compress_fused_kernel<<<(unsigned)grid, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace csa
