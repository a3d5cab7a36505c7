// decode_tc.cu -- decode-step lightning indexer and exact top-k (Hugging Face Transformers docs
// "DeepSeek-V4", section "Hybrid attention", CSA: the indexer scores the query against the
// compressed pool and keeps index_topk entries; the insight.ai.kr digest of the HF blog: ReLU
// multi-head dot product). One new query per sequence sees every one of its T cached entries:
//     I[b,s] = sum_h w[b,h] * ReLU(qI[b,h,:] . kI[b,s,:])
//
// The k^I stream (T x d_I bf16 per sequence: 8 MiB at 128K context, 64 MiB at 1M) dominates the
// step, so the score kernel is built to run at HBM speed: one persistent CTA per SM streams a
// contiguous range of k^I tiles through a 6-deep TMA ring (128-byte swizzle), the tensor cores form
// D[s,h] = kI[s,:] . qI[b,h,:] (entries on TMEM lanes, M=128 x N=HI), and each epilogue thread
// reduces its entry's HI heads in registers and writes one fp32 score.
//
// Top-k is exact and deterministic in two stages: every chunk of CHUNK scores keeps its own top-k
// (any entry of the global top-k is in its chunk's top-k under the same order), then one CTA per
// sequence selects the final k from the chunk candidates. Both stages are radix selects over
// order-preserving uint32 keys with ties to the smaller entry index; indices come out ascending.
#include <algorithm>

#include "kernels.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

constexpr int BM = 128;
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;
constexpr int MAX_STAGES = 6;
constexpr int NACC = 4;                // TMEM accumulators (each HI columns) in flight
constexpr int SEL_CHUNK = 8192;        // scores per first-stage select CTA
constexpr int SEL_THREADS = 512;
constexpr int MERGE_THREADS = 1024;

struct ScoreParams {
    const float *w;      // [B, HI]
    float *scores;       // [B, T]
    int32_t *status;
    int64_t T, G;        // entries per sequence; total tiles (B * tiles per sequence)
    int HI, dI, stages, tps;
};

// Persistent: CTA c takes the contiguous tile range [c*G/n, (c+1)*G/n) of the flat list
// (sequence-major, 128 entries per tile), so the HBM stream never idles on a wave tail. q^I of the
// current sequence is double-buffered; a range crosses at most a few sequence boundaries.
__global__ void __launch_bounds__(NUM_THREADS, 1)
decode_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        ScoreParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int kchunks = p.dI / 64;
    const uint32_t b_bytes = (uint32_t)kchunks * p.HI * 128;
    const uint32_t a_bytes = (uint32_t)kchunks * BM * 128;
    uint8_t *sB = smem;                                   // [2][b_bytes]
    uint8_t *sA = sB + 2 * b_bytes;
    float *sw = reinterpret_cast<float *>(sA + (size_t)p.stages * a_bytes);   // [HI] of the current sequence
    uint64_t *bars = reinterpret_cast<uint64_t *>(sw + 256);
    uint64_t *full = bars, *empty = bars + 8, *tfull = bars + 16, *tempty = bars + 20;   // tfull/tempty: [NACC]
    uint64_t *qfull = bars + 24, *qempty = bars + 26;     // [2] each
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 28);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 29);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g_lo = (int64_t)blockIdx.x * p.G / gridDim.x;
    const int64_t g_hi = (int64_t)(blockIdx.x + 1) * p.G / gridDim.x;
    const int ntiles = (int)(g_hi - g_lo);
    const int64_t b_first = g_lo / p.tps;
    const uint32_t tcols = p.HI * NACC <= 32 ? 32 : (p.HI * NACC <= 64 ? 64 : (p.HI * NACC <= 128 ? 128 : (p.HI * NACC <= 256 ? 256 : 512)));

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < NACC; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1);
            mbar_init(&qempty[i], 1);
        }
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (ntiles > 0) {
            const uint64_t pol_stream = policy_evict_first();   // k^I is read once per step
            int issued = 0, nseg = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int64_t g = g_lo + i, b = g / p.tps;
                const int it = (int)(g - b * p.tps), j = (int)(b - b_first);
                if (i == 0 || it == 0) {   // a new sequence: its q^I into buffer j & 1
                    if (!__all_sync(0xffffffffu, mbar_wait(&qempty[j & 1], ((j >> 1) & 1) ^ 1, abort, p.status))) break;
                    if (elect_one()) {
                        mbar_arrive_expect_tx(&qfull[j & 1], b_bytes);
                        for (int c = 0; c < kchunks; ++c)
                            tma_load_2d(sB + (j & 1) * b_bytes + c * p.HI * 128, &tm_q, &qfull[j & 1], c * 64,
                                        (int)(b * p.HI));
                    }
                    __syncwarp();
                    nseg = j + 1;
                }
                const int st = i % p.stages;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((i / p.stages) & 1) ^ 1, abort, p.status))) break;
                const int y = (int)(b * p.T + (int64_t)it * BM);
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[st], a_bytes);
                    for (int c = 0; c < kchunks; ++c)
                        tma_load_2d_hint(sA + st * a_bytes + c * BM * 128, &tm_k, &full[st], c * 64, y, pol_stream);
                }
                __syncwarp();
                issued = i + 1;
            }
            // never leave with copies in flight into this CTA's shared memory
            for (int j = max(0, nseg - 2); j < nseg; ++j)
                mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status, 100000000ull);
            for (int i = max(0, issued - p.stages); i < issued; ++i)
                mbar_wait(&full[i % p.stages], (i / p.stages) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp == 1) {
        if (ntiles > 0) {
            const uint32_t idesc = idesc_bf16(BM, p.HI);
            const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int64_t g = g_lo + i, b = g / p.tps;
                const int it = (int)(g - b * p.tps), j = (int)(b - b_first);
                if (i == 0 || it == 0)
                    if (!__all_sync(0xffffffffu, mbar_wait(&qfull[j & 1], (j >> 1) & 1, abort, p.status))) break;
                const int st = i % p.stages, buf = i % NACC;
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((i / NACC) & 1) ^ 1, abort, p.status))) break;
                if (!__all_sync(0xffffffffu, mbar_wait(&full[st], (i / p.stages) & 1, abort, p.status))) break;
                tc_fence_after();
                const uint64_t dBj = dB + (((j & 1) * b_bytes) >> 4);
                if (elect_one()) {   // one lane issues; the loop itself runs warp-wide (uniform operands)
                    for (int c = 0; c < kchunks; ++c)
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tmem + buf * p.HI, dA + ((st * a_bytes + c * BM * 128 + ks * 32) >> 4),
                                     dBj + ((c * p.HI * 128 + ks * 32) >> 4), idesc, (c | ks) != 0);
                    mma_commit(&empty[st]);
                    mma_commit(&tfull[buf]);
                    if (i + 1 == ntiles || it + 1 == p.tps) mma_commit(&qempty[j & 1]);   // done with this q^I
                }
                __syncwarp();
                issued = i + 1;
            }
            if (issued > 0)
                mbar_wait(&tfull[(issued - 1) % NACC], ((issued - 1) / NACC) & 1, abort, p.status, 100000000ull);
        }
    } else {
        const int quarter = warp & 3, etid = threadIdx.x - 64;
        const uint32_t taddr0 = tmem + ((uint32_t)(quarter * 32) << 16);
        float wr[64];   // index weights of the current sequence (HI == 64 keeps them in registers)
        for (int i = 0; i < ntiles; ++i) {
            const int64_t g = g_lo + i, b = g / p.tps;
            const int it = (int)(g - b * p.tps);
            if (i == 0 || it == 0) {   // index weights of the new sequence
                named_barrier_sync(1, EPI_THREADS);
                for (int h = etid; h < p.HI; h += EPI_THREADS) sw[h] = p.w[b * p.HI + h];
                named_barrier_sync(1, EPI_THREADS);
                if (p.HI == 64) {
#pragma unroll
                    for (int h = 0; h < 64; ++h) wr[h] = sw[h];
                }
            }
            const int buf = i % NACC;
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (i / NACC) & 1, abort, p.status))) break;
            tc_fence_after();
            float acc = 0.f;
            if (p.HI == 64) {
                float v0[32], v1[32];
                tmem_ld32(taddr0 + buf * 64, v0);        // both loads in flight, one wait
                tmem_ld32(taddr0 + buf * 64 + 32, v1);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&tempty[buf]);               // the accumulator may be reused from here
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    acc = fmaf(wr[jj], fmaxf(v0[jj], 0.f), acc);
                    acc = fmaf(wr[32 + jj], fmaxf(v1[jj], 0.f), acc);
                }
            } else {
                for (int h0 = 0; h0 < p.HI; h0 += 16) {
                    if (h0 + 32 <= p.HI) {
                        float v[32];
                        tmem_ld32(taddr0 + buf * p.HI + h0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 32; ++jj) acc = fmaf(sw[h0 + jj], fmaxf(v[jj], 0.f), acc);
                        h0 += 16;
                    } else {
                        float v[16];
                        tmem_ld16(taddr0 + buf * p.HI + h0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) acc = fmaf(sw[h0 + jj], fmaxf(v[jj], 0.f), acc);
                    }
                }
                tc_fence_before();
                mbar_arrive(&tempty[buf]);
            }
            const int64_t s = (int64_t)it * BM + quarter * 32 + lane;
            if (s < p.T) p.scores[b * p.T + s] = acc + 0.0f;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, tcols);
    }
}

// ---- block-level exact selection over keys in shared memory ------------------------------------------

// inclusive scan of one int per thread over the block; *total receives the block sum
__device__ __forceinline__ int block_incl_scan(int v, int *wsum, int *total)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) wsum[wid] = v;
    __syncthreads();
    if (wid == 0) {
        int x = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += n;
        }
        if (lane < nw) wsum[lane] = x;
    }
    __syncthreads();
    const int before = wid > 0 ? wsum[wid - 1] : 0;
    *total = wsum[nw - 1];
    __syncthreads();
    return v + before;
}

// Keep the k largest of keys[0..n) (ties: smaller position first). Writes the kept positions in
// ascending order to pos[0..min(k,n)) and returns that count. hist: 256 words; sh: 40 words.
// The radix digits start at the highest bit where the keys differ (scores of one query usually
// share sign and leading exponent bits, which would put every key into one or two bins).
__device__ int block_select(const uint32_t *keys, int n, int k, int *pos, uint32_t *hist, int *sh)
{
    if (n <= k) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) pos[i] = i;
        __syncthreads();
        return n;
    }
    // smallest and largest key
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        lo = min(lo, keys[i]);
        hi = max(hi, keys[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    uint32_t *red = reinterpret_cast<uint32_t *>(hist);   // 2 x 32 words of scratch before the passes
    if ((threadIdx.x & 31) == 0) {
        red[threadIdx.x >> 5] = lo;
        red[32 + (threadIdx.x >> 5)] = hi;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int nw = blockDim.x >> 5;
        uint32_t l2 = threadIdx.x < nw ? red[threadIdx.x] : 0xffffffffu;
        uint32_t h2 = threadIdx.x < nw ? red[32 + threadIdx.x] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            l2 = min(l2, __shfl_xor_sync(0xffffffffu, l2, o));
            h2 = max(h2, __shfl_xor_sync(0xffffffffu, h2, o));
        }
        if (threadIdx.x == 0) {
            sh[35] = (int)l2;
            sh[36] = (int)h2;
        }
    }
    __syncthreads();
    lo = (uint32_t)sh[35];
    hi = (uint32_t)sh[36];
    __syncthreads();
    uint32_t prefix, mask, remaining = (uint32_t)k;
    int lowbit;   // bits [0, lowbit) are still undecided
    if (lo == hi) {
        prefix = hi;
        mask = 0xffffffffu;
        lowbit = 0;
    } else {
        const int top = 31 - __clz(lo ^ hi);   // highest differing bit; bits above it are common
        mask = top == 31 ? 0u : ~((2u << top) - 1u);
        prefix = hi & mask;
        lowbit = top + 1;
    }
    while (lowbit > 0) {
        const int width = min(8, lowbit), shift = lowbit - width;
        const uint32_t dm = (1u << width) - 1u;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dm], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            uint32_t c[8], tot = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) { c[j] = hist[lane * 8 + j]; tot += c[j]; }
            uint32_t above = tot;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_down_sync(0xffffffffu, above, o);
                if (lane + o < 32) above += v;
            }
            above -= tot;
            int found = -1;
            uint32_t above_d = 0, cnt_d = 0, run = above;
#pragma unroll
            for (int j = 7; j >= 0; --j) {
                if (found < 0 && run + c[j] >= remaining) { found = lane * 8 + j; above_d = run; cnt_d = c[j]; }
                run += c[j];
            }
            if (found >= 0 && above < remaining) {
                sh[32] = found;
                sh[33] = (int)above_d;
                sh[34] = (int)cnt_d;
            }
        }
        __syncthreads();
        prefix |= (uint32_t)sh[32] << shift;
        mask |= dm << shift;
        remaining -= (uint32_t)sh[33];
        const bool whole_bucket = (uint32_t)sh[34] == remaining;
        lowbit = shift;
        __syncthreads();
        if (whole_bucket) break;
    }
    // ordered compaction: each thread owns a contiguous run of positions; two block scans place the
    // kept positions (keys above the threshold, and the first `remaining` equal ones) in order
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    const int b0 = min(n, (int)threadIdx.x * per), b1 = min(n, b0 + per);
    int ngt = 0, neq = 0;
    for (int i = b0; i < b1; ++i) {
        const uint32_t key = keys[i] & mask;
        ngt += key > prefix;
        neq += key == prefix;
    }
    int eq_tot;
    const int eq_before = block_incl_scan(neq, sh, &eq_tot) - neq;
    int take_eq = min(max((int)remaining - eq_before, 0), neq);
    const int cnt = ngt + take_eq;
    int total;
    int off = block_incl_scan(cnt, sh, &total) - cnt;
    for (int i = b0; i < b1; ++i) {
        const uint32_t key = keys[i] & mask;
        if (key > prefix || (key == prefix && take_eq-- > 0)) pos[off++] = i;
    }
    __syncthreads();
    return min(total, k);
}

// Stage 1: per (chunk of SEL_CHUNK scores, sequence) keep the chunk's top-k.
// cand_idx / cand_key: [B, nchunks, k] (entry index, key); unused slots hold -1 / 0.
__global__ void __launch_bounds__(SEL_THREADS)
topk_chunk_kernel(const float *__restrict__ scores, int64_t T, int k, int32_t *__restrict__ cand_idx,
                  uint32_t *__restrict__ cand_key)
{
    extern __shared__ uint32_t csm[];
    uint32_t *keys = csm;                                          // [SEL_CHUNK]
    int *pos = reinterpret_cast<int *>(csm + SEL_CHUNK);           // [SEL_CHUNK]
    __shared__ uint32_t hist[256];
    __shared__ int sh[40];
    const int b = blockIdx.y, nchunks = gridDim.x;
    const int64_t s0 = (int64_t)blockIdx.x * SEL_CHUNK;
    const int n = (int)min((int64_t)SEL_CHUNK, T - s0);
    const float *sc = scores + (int64_t)b * T + s0;
    for (int i = threadIdx.x; i < n; i += blockDim.x) keys[i] = score_key(sc[i]);
    __syncthreads();
    const int kk = min(k, SEL_CHUNK);
    const int cnt = block_select(keys, n, kk, pos, hist, sh);
    int32_t *oi = cand_idx + ((int64_t)b * nchunks + blockIdx.x) * k;
    uint32_t *ok = cand_key + ((int64_t)b * nchunks + blockIdx.x) * k;
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        if (j < cnt) {
            oi[j] = (int32_t)(s0 + pos[j]);
            ok[j] = keys[pos[j]];
        } else {
            oi[j] = -1;
            ok[j] = 0u;
        }
    }
}

// Stage 2: per sequence, the final top-k among the chunk candidates. Every chunk but the last
// holds exactly k candidates (k <= SEL_CHUNK), so the valid candidates are a prefix of the array,
// already in ascending entry order.
__global__ void __launch_bounds__(MERGE_THREADS)
topk_merge_kernel(const int32_t *__restrict__ cand_idx, const uint32_t *__restrict__ cand_key, int64_t T, int nchunks,
                  int k, int32_t *__restrict__ idx)
{
    extern __shared__ uint32_t msm[];
    __shared__ uint32_t hist[256];
    __shared__ int sh[40];
    const int b = blockIdx.x;
    const int total_max = nchunks * k;
    const int total = (nchunks - 1) * k + (int)min((int64_t)k, T - (int64_t)(nchunks - 1) * SEL_CHUNK);
    uint32_t *keys = msm;                                         // [total_max]
    int *ids = reinterpret_cast<int *>(msm + total_max);          // [total_max]
    int *pos = ids + total_max;                                   // [total_max]
    const int32_t *ci = cand_idx + (int64_t)b * total_max;
    const uint32_t *ck = cand_key + (int64_t)b * total_max;
    for (int j = threadIdx.x; j < total; j += blockDim.x) {
        keys[j] = ck[j];
        ids[j] = ci[j];
    }
    __syncthreads();
    const int cnt = block_select(keys, total, k, pos, hist, sh);
    int32_t *out = idx + (int64_t)b * k;
    for (int j = threadIdx.x; j < k; j += blockDim.x) out[j] = j < cnt ? ids[pos[j]] : -1;
}

}  // namespace

size_t decode_index_workspace(int64_t B, int64_t T, int k)
{
    const int64_t nchunks = (T + SEL_CHUNK - 1) / SEL_CHUNK;
    return (size_t)B * T * 4 + 2 * (size_t)B * nchunks * k * 4 + 1024;
}

bool decode_index_tc_supported(int64_t T, int HI, int dI, int k)
{
    const int64_t nchunks = (T + SEL_CHUNK - 1) / SEL_CHUNK;
    return (dI == 64 || dI == 128) && (HI == 16 || HI == 32 || HI == 64 || HI == 128) && T >= 1 && k >= 1 &&
           k <= SEL_CHUNK && nchunks * k * 12 <= 200 * 1024 && T <= (1ll << 26);
}

// scores/candidates live in `ws` (decode_index_workspace bytes, 256-byte aligned)
cudaError_t launch_decode_index_tc(const uint16_t *qI, const float *w, const uint16_t *kI, int64_t B, int64_t T, int HI,
                                   int dI, int k, int32_t *idx, void *ws, int32_t *status, cudaStream_t stream)
{
    if (B == 0) return cudaSuccess;
    char *p8 = static_cast<char *>(ws);
    float *scores = reinterpret_cast<float *>(p8);
    const int64_t nchunks = (T + SEL_CHUNK - 1) / SEL_CHUNK;
    const size_t sbytes = ((size_t)B * T * 4 + 255) & ~(size_t)255;
    int32_t *cand_idx = reinterpret_cast<int32_t *>(p8 + sbytes);
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(p8 + sbytes + (size_t)B * nchunks * k * 4);

    CUtensorMap tq, tk;
    if (!make_tmap_bf16_sw128(&tq, qI, (uint64_t)B * HI, dI, HI)) return cudaErrorInvalidValue;
    if (!make_tmap_bf16_sw128(&tk, kI, (uint64_t)(B * T), dI, BM)) return cudaErrorInvalidValue;
    ScoreParams sp;
    sp.w = w;
    sp.scores = scores;
    sp.status = status;
    sp.T = T;
    sp.HI = HI;
    sp.dI = dI;
    sp.tps = (int)((T + BM - 1) / BM);
    sp.G = (int64_t)B * sp.tps;
    const size_t a_bytes = (size_t)(dI / 64) * BM * 128;
    const size_t fixed = 1024 + 2 * (size_t)(dI / 64) * HI * 128 + 256 * 4 + 256;
    sp.stages = (int)std::min<size_t>(MAX_STAGES, (227 * 1024 - fixed) / a_bytes);
    const size_t smem = fixed + (size_t)sp.stages * a_bytes;
    cudaError_t e = cudaFuncSetAttribute(decode_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const unsigned g1 = (unsigned)std::min<int64_t>(nsm, sp.G);
    decode_scores_tc_kernel<<<g1, NUM_THREADS, smem, stream>>>(tq, tk, sp);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    dim3 g2((unsigned)nchunks, (unsigned)B);
    const size_t csmem = (size_t)SEL_CHUNK * 8;
    e = cudaFuncSetAttribute(topk_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)csmem);
    if (e != cudaSuccess) return e;
    topk_chunk_kernel<<<g2, SEL_THREADS, csmem, stream>>>(scores, T, k, cand_idx, cand_key);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t msmem = (size_t)nchunks * k * 12;
    e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
    topk_merge_kernel<<<(unsigned)B, MERGE_THREADS, msmem, stream>>>(cand_idx, cand_key, T, (int)nchunks, k, idx);
    return cudaGetLastError();
}

}  // namespace csa
