// decode_tc.cu -- decode-step lightning indexer and exact top-k (Hugging Face Transformers docs
// "DeepSeek-V4", section "Hybrid attention", CSA: the indexer scores the query against the
// compressed pool and keeps index_topk entries; the insight.ai.kr digest of the HF blog: ReLU
// multi-head dot product). One new query per sequence sees every one of its T cached entries:
//     I[b,s] = sum_h w[b,h] * ReLU(qI[b,h,:] . kI[b,s,:])
//
// The k^I stream (T x d_I bf16 per sequence: 8 MiB at 128K context, 64 MiB at 1M) dominates the
// step, so the score kernel is built to run at HBM speed: each CTA streams a contiguous chunk of
// one sequence's k^I through a 6-deep TMA ring (128-byte swizzle), the tensor cores form
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
constexpr int SCORE_CHUNK = 4096;      // entries per score CTA
constexpr int SEL_CHUNK = 8192;        // scores per first-stage select CTA
constexpr int SEL_THREADS = 512;
constexpr int MERGE_THREADS = 1024;

struct ScoreParams {
    const float *w;      // [B, HI]
    float *scores;       // [B, T]
    int32_t *status;
    int64_t T;
    int HI, dI, stages;
};

__global__ void __launch_bounds__(NUM_THREADS, 1)
decode_scores_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        ScoreParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int kchunks = p.dI / 64;
    const uint32_t b_bytes = (uint32_t)kchunks * p.HI * 128;
    const uint32_t a_bytes = (uint32_t)kchunks * BM * 128;
    uint8_t *sB = smem;
    uint8_t *sA = sB + b_bytes;
    float *sw = reinterpret_cast<float *>(sA + (size_t)p.stages * a_bytes);   // [HI]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sw + 256);
    uint64_t *full = bars, *empty = bars + 8, *tfull = bars + 16, *tempty = bars + 18, *qfull = bars + 20;
    uint32_t *tmem_ptr = reinterpret_cast<uint32_t *>(bars + 21);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 22);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int64_t s_begin = (int64_t)blockIdx.x * SCORE_CHUNK;
    const int64_t s_end = min(p.T, s_begin + SCORE_CHUNK);
    const int ntiles = (int)((s_end - s_begin + BM - 1) / BM);
    const uint32_t tcols = p.HI * 2 <= 32 ? 32 : (p.HI * 2 <= 64 ? 64 : (p.HI * 2 <= 128 ? 128 : 256));

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], EPI_THREADS); }
        mbar_init(qfull, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_ptr, tcols);
        tmem_relinquish();
    }
    if (warp >= 2)
        for (int i = threadIdx.x - 64; i < p.HI; i += EPI_THREADS) sw[i] = p.w[(int64_t)b * p.HI + i];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;

    if (warp == 0) {
        if (elect_one() && ntiles > 0) {
            const uint64_t pol_stream = policy_evict_first();   // k^I is read once per step
            mbar_arrive_expect_tx(qfull, b_bytes);
            for (int c = 0; c < kchunks; ++c) tma_load_2d(sB + c * p.HI * 128, &tm_q, qfull, c * 64, b * p.HI);
            int issued = 0;
            for (int i = 0; i < ntiles; ++i) {
                const int st = i % p.stages;
                if (!mbar_wait(&empty[st], ((i / p.stages) & 1) ^ 1, abort, p.status)) break;
                mbar_arrive_expect_tx(&full[st], a_bytes);
                const int y = (int)((int64_t)b * p.T + s_begin + (int64_t)i * BM);
                for (int c = 0; c < kchunks; ++c)
                    tma_load_2d_hint(sA + st * a_bytes + c * BM * 128, &tm_k, &full[st], c * 64, y, pol_stream);
                issued = i + 1;
            }
            mbar_wait(qfull, 0, abort, p.status, 100000000ull);
            for (int i = max(0, issued - p.stages); i < issued; ++i)
                mbar_wait(&full[i % p.stages], (i / p.stages) & 1, abort, p.status, 100000000ull);
        }
    } else if (warp == 1) {
        if (lane == 0 && ntiles > 0) {
            const uint32_t idesc = idesc_bf16(BM, p.HI);
            const uint64_t dA = sdesc_sw128(smem_u32(sA), 16, 1024), dB = sdesc_sw128(smem_u32(sB), 16, 1024);
            bool ok = mbar_wait(qfull, 0, abort, p.status);
            int issued = 0;
            for (int i = 0; ok && i < ntiles; ++i) {
                const int st = i % p.stages, buf = i & 1;
                if (!mbar_wait(&tempty[buf], ((i >> 1) & 1) ^ 1, abort, p.status)) break;
                if (!mbar_wait(&full[st], (i / p.stages) & 1, abort, p.status)) break;
                tc_fence_after();
                for (int c = 0; c < kchunks; ++c)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_bf16(tmem + buf * p.HI, dA + ((st * a_bytes + c * BM * 128 + ks * 32) >> 4),
                                 dB + ((c * p.HI * 128 + ks * 32) >> 4), idesc, (c | ks) != 0);
                mma_commit(&empty[st]);
                mma_commit(&tfull[buf]);
                issued = i + 1;
            }
            if (issued > 0) mbar_wait(&tfull[(issued - 1) & 1], ((issued - 1) >> 1) & 1, abort, p.status, 100000000ull);
        }
    } else {
        const int quarter = warp & 3;
        const uint32_t taddr0 = tmem + ((uint32_t)(quarter * 32) << 16);
        for (int i = 0; i < ntiles; ++i) {
            const int buf = i & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (i >> 1) & 1, abort, p.status))) break;
            tc_fence_after();
            float acc = 0.f;
            for (int h0 = 0; h0 < p.HI; h0 += 16) {
                if (h0 + 32 <= p.HI) {
                    float v[32];
                    tmem_ld32(taddr0 + buf * p.HI + h0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc = fmaf(sw[h0 + j], fmaxf(v[j], 0.f), acc);
                    h0 += 16;
                } else {
                    float v[16];
                    tmem_ld16(taddr0 + buf * p.HI + h0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc = fmaf(sw[h0 + j], fmaxf(v[j], 0.f), acc);
                }
            }
            tc_fence_before();
            mbar_arrive(&tempty[buf]);
            const int64_t s = s_begin + (int64_t)i * BM + quarter * 32 + lane;
            if (s < s_end) p.scores[(int64_t)b * p.T + s] = acc + 0.0f;
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
__device__ int block_select(const uint32_t *keys, int n, int k, int *pos, uint32_t *hist, int *sh)
{
    if (n <= k) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) pos[i] = i;
        __syncthreads();
        return n;
    }
    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += blockDim.x) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
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
        mask |= 255u << shift;
        remaining -= (uint32_t)sh[33];
        const bool whole_bucket = (uint32_t)sh[34] == remaining;
        __syncthreads();
        if (whole_bucket) break;
    }
    int written = 0, eq_seen = 0;
    for (int base = 0; base < n; base += blockDim.x) {
        const int i = base + threadIdx.x;
        const uint32_t key = i < n ? (keys[i] & mask) : 0u;
        const int is_eq = (i < n && key == prefix) ? 1 : 0;
        int eq_tot;
        const int eq_incl = block_incl_scan(is_eq, sh, &eq_tot);
        const int rank = eq_seen + eq_incl - is_eq;
        const int sel = (i < n && (key > prefix || (is_eq && rank < (int)remaining))) ? 1 : 0;
        int sel_tot;
        const int sel_incl = block_incl_scan(sel, sh, &sel_tot);
        if (sel) pos[written + sel_incl - 1] = i;
        written += sel_tot;
        eq_seen += eq_tot;
        if (written >= k) break;
    }
    __syncthreads();
    return written;
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
    const size_t a_bytes = (size_t)(dI / 64) * BM * 128;
    const size_t fixed = 1024 + (size_t)(dI / 64) * HI * 128 + 256 * 4 + 256;
    sp.stages = (int)std::min<size_t>(MAX_STAGES, (227 * 1024 - fixed) / a_bytes);
    const size_t smem = fixed + (size_t)sp.stages * a_bytes;
    cudaError_t e = cudaFuncSetAttribute(decode_scores_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 g1((unsigned)((T + SCORE_CHUNK - 1) / SCORE_CHUNK), (unsigned)B);
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
