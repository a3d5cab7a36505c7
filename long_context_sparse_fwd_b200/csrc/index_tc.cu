// index_tc.cu -- lightning indexer on the 5th-generation tensor cores with the top-k fused in.
//
// Scores (Hugging Face Transformers docs "DeepSeek-V4", section "Hybrid attention", CSA; the
// insight.ai.kr digest of the HF blog: a ReLU multi-head dot product):
//     I[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:]),   s < vis(t) = floor((t+1)/m)
// then the top-k per query with ties to the smaller entry index ("Attention mask layout":
// unfilled slots are -1).
//
// Mapping: the GEMM is transposed so an entry sits on a TMEM lane and the (query, head) pairs of
// Q = 256/HI consecutive queries run along the N = 256 columns:
//     D[s, (q,h)] = kI[s,:] . qI[q,h,:]          M = 128 entries, N = 256, K = dI
// Each epilogue thread then owns one entry and reduces a query's HI columns in registers
// (w-weighted ReLU sum): no cross-lane reduction. The scores of the Q queries for every visible
// entry stay in shared memory; once a group's last entry tile is scored, a pair of warps per query
// runs the exact selection and writes the kept indices in ascending order.
//
// Persistent: one CTA per SM walks groups of Q queries, the groups that see the most entries first.
// Roles (18 warps): warp 0 issues TMA loads (a group's q^I block, then its k^I tiles through a ring
// of stages), warp 1 owns TMEM (2 x 256 columns, double-buffered accumulators) and issues
// tcgen05.mma, warps 2-9 read TMEM and score (two warps per lane quarter, each half of the
// queries), warps 10-17 (four pairs) select the previous group's top-k from a second scores buffer
// while the next group is scored. Every wait is bounded; a timeout sets CSA_ERR_TIMEOUT.
#include <algorithm>

#include "kernels.cuh"
#include "sm100.cuh"

namespace csa {

using namespace sm100;

namespace {

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

constexpr int BM = 128;          // entries per tile = TMEM lanes
constexpr int BN = 256;          // (query, head) columns
constexpr int EPI_THREADS = 256;       // warps 2-9: two warps per TMEM lane quarter, each half of the queries
constexpr int TOPK_THREADS = 256;      // warps 10-17: four pairs, one query each at a time
constexpr int NUM_THREADS = 64 + EPI_THREADS + TOPK_THREADS;
constexpr uint32_t TMEM_COLS = 512;

struct IdxParams {
    const float *w;      // [S, HI]
    int32_t *idx;        // [S, k]
    int32_t *status;
    int64_t S, T;
    int64_t pos0;        // position of query row 0
    int64_t ngroups;     // groups of Q consecutive queries
    int HI, dI, m, k, Q, stages, T_cap;
    int nsb;             // scores buffers (2: the top-k of a group overlaps the next group's scoring)
    int bn;              // (query, head) columns per group: 256 (bf16), 128 (MXFP4)
    // Entries are scored in chunks of `chunk` (a multiple of 128). One chunk covering every entry
    // (kcap = 0) is ranked in place. Otherwise each query's scores buffer holds its running top-k
    // (up to kcap scores) right before the chunk's scores, so the ranking of [running set, chunk]
    // keeps the running set exact; qstride = kcap + chunk floats per query.
    int chunk, kcap, qstride;
    // MXFP4 operands (fp4 != 0): q^I and k^I as packed E2M1 codes (the tensor maps) with one E8M0
    // scale per 32 channels: qs [S, HI, 4], ks [T, 4] (d_I = 128)
    int fp4;
    const uint8_t *qs, *ks;
};

// Scale-factor columns of the MXFP4 mode (after the two 128-column accumulators): per accumulator
// buffer a k^I slot, per group parity a q^I slot, 4 columns each.
constexpr uint32_t F4_SFA_COL = 256, F4_SFB_COL = 264;

// Exact top-k of one query's scores by one warp: radix select over order-preserving keys, starting
// at the highest bit where the keys differ (one query's scores usually share their leading bits), then
// one ordered pass that keeps the selected indices in ascending order (ties to the smaller index).
__device__ __forceinline__ void topk_warp(const float *sc, int n, int k, uint32_t *hist, int32_t *out)
{
    const int lane = threadIdx.x & 31;
    if (n <= k) {
        for (int i = lane; i < k; i += 32) out[i] = i < n ? i : -1;
        return;
    }
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int s = lane; s < n; s += 32) {
        const uint32_t key = score_key(sc[s]);
        lo = min(lo, key);
        hi = max(hi, key);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    uint32_t prefix, mask, remaining = (uint32_t)k;
    int lowbit;
    if (lo == hi) {
        prefix = hi;
        mask = 0xffffffffu;
        lowbit = 0;
    } else {
        const int top = 31 - __clz(lo ^ hi);
        mask = top == 31 ? 0u : ~((2u << top) - 1u);
        prefix = hi & mask;
        lowbit = top + 1;
    }
    while (lowbit > 0) {
        const int width = min(8, lowbit), shift = lowbit - width;
        const uint32_t dm = (1u << width) - 1u;
#pragma unroll
        for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
        __syncwarp();
        for (int s = lane; s < n; s += 32) {
            const uint32_t key = score_key(sc[s]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dm], 1u);
        }
        __syncwarp();
        uint32_t c[8], tot = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) { c[j] = hist[lane * 8 + j]; tot += c[j]; }
        uint32_t above = tot;   // counts held by higher lanes (higher digits)
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
        const unsigned who = __ballot_sync(0xffffffffu, found >= 0 && (above < remaining));
        const int src = __ffs(who) - 1;
        const int d = __shfl_sync(0xffffffffu, found, src);
        above_d = __shfl_sync(0xffffffffu, above_d, src);
        cnt_d = __shfl_sync(0xffffffffu, cnt_d, src);
        prefix |= (uint32_t)d << shift;
        mask |= dm << shift;
        remaining -= above_d;
        lowbit = shift;
        __syncwarp();
        if (cnt_d == remaining) break;   // the whole bucket is taken
    }
    int written = 0, eq_seen = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n && written < k; base += 32) {
        const int s = base + lane;
        uint32_t key = 0;
        if (s < n) key = score_key(sc[s]) & mask;
        const bool gt = s < n && key > prefix;
        const bool eq = s < n && key == prefix;
        const unsigned eqb = __ballot_sync(0xffffffffu, eq);
        const int rank = eq_seen + __popc(eqb & lt);
        const bool sel = gt || (eq && rank < (int)remaining);
        const unsigned sb = __ballot_sync(0xffffffffu, sel);
        if (sel) out[written + __popc(sb & lt)] = s;
        written += __popc(sb);
        eq_seen += __popc(eqb);
    }
    for (int i = written + lane; i < k; i += 32) out[i] = -1;
}


// Exact top-k of one query's scores by a pair of warps (64 threads, named barrier `bar`), ties to the
// smaller index, indices written in ascending order. A histogram of the (up to) 10 key bits below
// the highest bit where the query's keys differ gives the threshold bin; its entries are ranked
// (key descending, index ascending) to find the last selected (key, index); one ordered pass then
// writes every entry that beats or equals it. A threshold bin of more than 512 entries falls back to
// the single-warp radix select. `scratch`: 4 KB (histogram, then the bin's entries) + 80 words.
constexpr int PBINS = 1024;
constexpr int PCAND = 512;

__device__ __forceinline__ void pair_sync(int bar) { named_barrier_sync(bar, 64); }

__device__ void topk_pair(const float *sc, int n, int k, uint32_t *scratch, int bar, int32_t *out)
{
    const int pt = threadIdx.x & 63, lane = threadIdx.x & 31, pw = pt >> 5;
    uint32_t *hist = scratch;                                  // [PBINS]
    uint2 *cand = reinterpret_cast<uint2 *>(scratch);          // [PCAND] after the threshold is known
    uint32_t *vars = scratch + PBINS;                          // [16]
    if (n <= k) {
        for (int i = pt; i < k; i += 64) out[i] = i < n ? i : -1;
        return;
    }
    // key range
    uint32_t lo = 0xffffffffu, hi = 0u;
    for (int i = pt; i < n; i += 64) {
        const uint32_t key = score_key(sc[i]);
        lo = min(lo, key);
        hi = max(hi, key);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    for (int i = pt; i < PBINS; i += 64) hist[i] = 0u;
    if (lane == 0) {
        vars[2 * pw] = lo;
        vars[2 * pw + 1] = hi;
    }
    pair_sync(bar);
    lo = min(vars[0], vars[2]);
    hi = max(vars[1], vars[3]);
    const uint32_t diff = lo ^ hi;
    int shift = 0;
    uint32_t dmask = 0u;
    if (diff != 0u) {
        const int top = 31 - __clz(diff);
        shift = max(0, top - 9);
        dmask = (2u << (top - shift)) - 1u;
    }
    for (int i = pt; i < n; i += 64) atomicAdd(&hist[(score_key(sc[i]) >> shift) & dmask], 1u);
    pair_sync(bar);
    // threshold bin: thread pt owns bins [16 pt, 16 pt + 16); suffix sums over the owners
    uint32_t own = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) own += hist[16 * pt + j];
    uint32_t after = own;   // owners above this one, within the warp
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_down_sync(0xffffffffu, after, o);
        if (lane + o < 32) after += x;
    }
    after -= own;
    if (lane == 0) vars[4 + pw] = after + own;   // this warp's total
    pair_sync(bar);
    if (pw == 0) after += vars[5];               // warp 1 owns the higher bins
    {
        uint32_t run = after;
        for (int j = 15; j >= 0; --j) {
            const uint32_t c = hist[16 * pt + j];
            if (run < (uint32_t)k && run + c >= (uint32_t)k) {
                vars[6] = (uint32_t)(16 * pt + j);   // d*
                vars[7] = run;                       // entries in higher bins
            }
            run += c;
        }
    }
    if (pt == 0) vars[8] = 0u;   // candidate count
    pair_sync(bar);
    const uint32_t dstar = vars[6], above = vars[7], remaining = (uint32_t)k - above;
    // entries of the threshold bin
    for (int base = pw * 32; base < n; base += 64) {
        const int i = base + lane;
        uint32_t key = 0u;
        bool isc = false;
        if (i < n) {
            key = score_key(sc[i]);
            isc = ((key >> shift) & dmask) == dstar;
        }
        const unsigned m = __ballot_sync(0xffffffffu, isc);
        if (m != 0u) {
            uint32_t pos0 = 0;
            if (lane == 0) pos0 = atomicAdd(&vars[8], (uint32_t)__popc(m));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            const uint32_t pos = pos0 + __popc(m & ((1u << lane) - 1u));
            if (isc && pos < (uint32_t)PCAND) cand[pos] = make_uint2(key, (uint32_t)i);
        }
    }
    pair_sync(bar);
    const uint32_t nc = vars[8];
    if (nc > (uint32_t)PCAND) {   // crowded bin: the single-warp radix select (exact)
        if (pw == 0) topk_warp(sc, n, k, scratch, out);
        pair_sync(bar);            // the scratch is free again for the pair's next query
        return;
    }
    // the remaining-th best entry of the bin: rank = number of entries that beat it
    for (uint32_t c = pt; c < nc; c += 64) {
        const uint2 me = cand[c];
        uint32_t rank = 0;
        for (uint32_t j = 0; j < nc; ++j) {
            const uint2 o = cand[j];
            rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
        }
        if (rank == remaining - 1u) {
            vars[9] = me.x;
            vars[10] = me.y;
        }
    }
    pair_sync(bar);
    const uint32_t tkey = vars[9], tidx = vars[10];
    // ordered output: warp 0 takes entries [0, half), warp 1 [half, n); warp 1 starts after warp 0's count
    const int half = (((n + 1) >> 1) + 31) & ~31;
    const int b0 = pw == 0 ? 0 : min(half, n), b1 = pw == 0 ? min(half, n) : n;
    const unsigned lt = (1u << lane) - 1u;
    int cnt = 0;
    for (int base = b0; base < b1; base += 32) {
        const int i = base + lane;
        bool sel = false;
        if (i < b1) {
            const uint32_t key = score_key(sc[i]);
            sel = key > tkey || (key == tkey && (uint32_t)i <= tidx);
        }
        cnt += __popc(__ballot_sync(0xffffffffu, sel));
    }
    if (pw == 0 && lane == 0) vars[11] = (uint32_t)cnt;
    pair_sync(bar);
    int written = pw == 0 ? 0 : (int)vars[11];
    for (int base = b0; base < b1; base += 32) {
        const int i = base + lane;
        bool sel = false;
        if (i < b1) {
            const uint32_t key = score_key(sc[i]);
            sel = key > tkey || (key == tkey && (uint32_t)i <= tidx);
        }
        const unsigned sb = __ballot_sync(0xffffffffu, sel);
        if (sel) out[written + __popc(sb & lt)] = i;
        written += __popc(sb);
    }
    pair_sync(bar);
}

// As topk_pair for n <= 2048 with the keys held in registers: thread pt of the pair holds entries
// pt + 64 j (j < 32), so every pass is an unrolled loop over registers, and warp pw holds the
// 32-entry groups g = 2 j + pw in index order for the ordered output.
__device__ void topk_pair_reg(const float *sc, int n, int k, uint32_t *scratch, int bar, int32_t *out)
{
    constexpr int KPT = 32;
    const int pt = threadIdx.x & 63, lane = threadIdx.x & 31, pw = pt >> 5;
    uint32_t *hist = scratch;                                  // [PBINS]
    uint2 *cand = reinterpret_cast<uint2 *>(scratch);          // [PCAND] after the threshold is known
    uint32_t *vars = scratch + PBINS;                          // [16]
    uint32_t key[KPT];
    uint32_t lo = 0xffffffffu, hi = 0u;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int i = pt + 64 * j;
        key[j] = i < n ? score_key(sc[i]) : 0u;
        if (i < n) {
            lo = min(lo, key[j]);
            hi = max(hi, key[j]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, o));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    for (int i = pt; i < PBINS; i += 64) hist[i] = 0u;
    if (lane == 0) {
        vars[2 * pw] = lo;
        vars[2 * pw + 1] = hi;
    }
    pair_sync(bar);
    lo = min(vars[0], vars[2]);
    hi = max(vars[1], vars[3]);
    const uint32_t diff = lo ^ hi;
    int shift = 0;
    uint32_t dmask = 0u;
    if (diff != 0u) {
        const int top = 31 - __clz(diff);
        shift = max(0, top - 9);
        dmask = (2u << (top - shift)) - 1u;
    }
#pragma unroll
    for (int j = 0; j < KPT; ++j)
        if (pt + 64 * j < n) atomicAdd(&hist[(key[j] >> shift) & dmask], 1u);
    pair_sync(bar);
    uint32_t hv[16], own = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        hv[j] = hist[16 * pt + j];
        own += hv[j];
    }
    uint32_t after = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t x = __shfl_down_sync(0xffffffffu, after, o);
        if (lane + o < 32) after += x;
    }
    after -= own;
    if (lane == 0) vars[4 + pw] = after + own;
    pair_sync(bar);
    if (pw == 0) after += vars[5];
    {
        uint32_t run = after;
#pragma unroll
        for (int j = 15; j >= 0; --j) {
            if (run < (uint32_t)k && run + hv[j] >= (uint32_t)k) {
                vars[6] = (uint32_t)(16 * pt + j);
                vars[7] = run;
            }
            run += hv[j];
        }
    }
    if (pt == 0) vars[8] = 0u;
    pair_sync(bar);
    const uint32_t dstar = vars[6], remaining = (uint32_t)k - vars[7];
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int i = pt + 64 * j;
        const bool isc = i < n && ((key[j] >> shift) & dmask) == dstar;
        const unsigned m = __ballot_sync(0xffffffffu, isc);
        if (m != 0u) {
            uint32_t pos0 = 0;
            if (lane == 0) pos0 = atomicAdd(&vars[8], (uint32_t)__popc(m));
            pos0 = __shfl_sync(0xffffffffu, pos0, 0);
            const uint32_t pos = pos0 + __popc(m & ((1u << lane) - 1u));
            if (isc && pos < (uint32_t)PCAND) cand[pos] = make_uint2(key[j], (uint32_t)i);
        }
    }
    pair_sync(bar);
    const uint32_t nc = vars[8];
    if (nc > (uint32_t)PCAND) {   // crowded bin: the single-warp radix select (exact)
        if (pw == 0) topk_warp(sc, n, k, scratch, out);
        pair_sync(bar);
        return;
    }
    for (uint32_t c = pt; c < nc; c += 64) {
        const uint2 me = cand[c];
        uint32_t rank = 0;
        for (uint32_t j = 0; j < nc; ++j) {
            const uint2 o = cand[j];
            rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
        }
        if (rank == remaining - 1u) {
            vars[9] = me.x;
            vars[10] = me.y;
        }
    }
    pair_sync(bar);
    const uint32_t tkey = vars[9], tidx = vars[10];
    // ordered output: group counts of this warp's groups (g = 2 j + pw), exclusive scan over all 64
    uint32_t *gcnt = scratch + PBINS + 16;   // [64] (scratch tail, past vars)
    unsigned selm[KPT];
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int i = pt + 64 * j;
        const bool sel = i < n && (key[j] > tkey || (key[j] == tkey && (uint32_t)i <= tidx));
        selm[j] = __ballot_sync(0xffffffffu, sel);
        if (lane == 0) gcnt[2 * j + pw] = (uint32_t)__popc(selm[j]);
    }
    pair_sync(bar);
    if (pw == 0) {   // exclusive scan of the 64 group counts (two per lane)
        const uint32_t c0 = gcnt[2 * lane], c1 = gcnt[2 * lane + 1];
        uint32_t incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t x = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += x;
        }
        const uint32_t excl = incl - (c0 + c1);
        gcnt[2 * lane] = excl;
        gcnt[2 * lane + 1] = excl + c0;
    }
    pair_sync(bar);
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < KPT; ++j) {
        const int i = pt + 64 * j;
        if ((selm[j] >> lane) & 1u) out[gcnt[2 * j + pw] + __popc(selm[j] & lt)] = i;
    }
    pair_sync(bar);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
index_topk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     IdxParams p)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int kchunks = p.dI / 64;                      // 128-byte swizzle atoms along K (bf16)
    // bf16: 128-byte swizzled rows of 64 channels; MXFP4: one 64-byte swizzled row of 128 packed codes
    const uint32_t b_bytes = p.fp4 ? (uint32_t)p.bn * 64 : (uint32_t)kchunks * BN * 128;
    const uint32_t a_bytes = p.fp4 ? (uint32_t)BM * 64 : (uint32_t)kchunks * BM * 128;
    uint8_t *sB = smem;
    uint8_t *sA = sB + b_bytes;
    float *scores_all = reinterpret_cast<float *>(sA + (size_t)p.stages * a_bytes);   // [nsb][Q][qstride]
    float *sw = scores_all + (size_t)p.nsb * p.Q * p.qstride;                        // [BN]
    uint32_t *hist = reinterpret_cast<uint32_t *>(sw + BN);                          // [4 pairs][PBINS + 80]
    // MXFP4: k^I scales of every tile [T_cap / 128][32 x 16 bytes] and the group's q^I scales [2][32 x 16]
    // in the arrangement the scale copy into TMEM takes (row r: the scale words of rows r + 32 j)
    // chunked ranking: running top-k of each query (scores, entry indices, count) and each pair's
    // selected positions
    float *run_sc = reinterpret_cast<float *>(hist + 4 * (PBINS + 80));              // [Q][kcap]
    int32_t *run_idx = reinterpret_cast<int32_t *>(run_sc + (size_t)p.Q * p.kcap);     // [Q][kcap]
    int32_t *run_cnt = run_idx + (size_t)p.Q * p.kcap;                                 // [Q] (16-aligned)
    int32_t *sel_all = run_cnt + ((p.kcap > 0 ? p.Q : 0) + 3) / 4 * 4;                 // [4 pairs][kcap]
    uint8_t *sSFA = reinterpret_cast<uint8_t *>(sel_all + 4 * (size_t)p.kcap);
    uint8_t *sSFB = sSFA + (p.fp4 ? (size_t)(p.T_cap / BM) * 512 : 0);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSFB + (p.fp4 ? 1024 : 0));
    uint64_t *full = bars;                   // [stages] k^I tile landed
    uint64_t *empty = bars + 8;              // [stages] its MMAs completed
    uint64_t *tfull = bars + 16;             // [2] accumulator written
    uint64_t *tempty = bars + 18;            // [2] accumulator read by the 256 epilogue threads
    uint64_t *qfull = bars + 20;             // q^I of the group landed
    uint64_t *qempty = bars + 21;            // every MMA of the group completed: q^I may be replaced
    uint64_t *sfull = bars + 22;             // [2] scores buffer complete (8 epilogue warps)
    uint64_t *sempty = bars + 24;            // [2] scores buffer consumed by the top-k (8 warps)
    uint32_t *tmem_base_ptr = reinterpret_cast<uint32_t *>(bars + 26);
    volatile int *abort = reinterpret_cast<volatile int *>(bars + 27);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Groups of Q consecutive queries, the ones that see the most entries first, dealt round-robin.
    auto group_of = [&](int64_t gi, int64_t *t0, int *ntiles) -> bool {
        const int64_t G = blockIdx.x + gi * gridDim.x;
        if (G >= p.ngroups) return false;
        *t0 = (p.ngroups - 1 - G) * p.Q;
        const int64_t t_last = min(*t0 + p.Q - 1, p.S - 1);
        *ntiles = (int)((visible_entries(p.pos0 + t_last, p.m, p.T) + BM - 1) / BM);
        return true;
    };

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tfull[i], 1);
            mbar_init(&tempty[i], EPI_THREADS);
            mbar_init(&sfull[i], EPI_THREADS / 32);
            mbar_init(&sempty[i], TOPK_THREADS / 32);
        }
        mbar_init(qfull, p.fp4 ? 2 : 1);   // MXFP4: the code load and the gathered q^I scales
        mbar_init(qempty, 1);
        *abort = 0;
        fence_barrier_init();
    }
    if (p.fp4) {   // every tile's k^I scales, once: tile t, row r, word j = the scale word of entry 128 t + r + 32 j
        const int nwords = p.T_cap;
        for (int e = threadIdx.x; e < nwords; e += NUM_THREADS) {
            const uint32_t v = e < p.T ? *reinterpret_cast<const uint32_t *>(p.ks + (int64_t)e * 4) : 0u;
            const int t = e / BM, rr = e % BM;
            *reinterpret_cast<uint32_t *>(sSFA + t * 512 + (rr & 31) * 16 + (rr >> 5) * 4) = v;
        }
        fence_async_smem();   // read by tcgen05.cp through the async proxy
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_ptr, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_ptr;

    if (warp == 0) {
        // ---------------- TMA producer (warp-wide loop, one elected lane issues) ----------------
        if (elect_one()) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_k);
        }
        __syncwarp();
        int tile = 0, issued = 0;
        int64_t ngr = 0;
        bool ok = true;
        int64_t t0;
        int ntiles;
        for (int64_t gi = 0; ok && group_of(gi, &t0, &ntiles); ++gi) {
            // q^I of this group once every MMA of the previous group has completed
            if (gi > 0 && !__all_sync(0xffffffffu, mbar_wait(qempty, (uint32_t)((gi - 1) & 1), abort, p.status))) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(qfull, b_bytes);
                if (p.fp4) {
                    tma_load_2d(sB, &tm_q, qfull, 0, (int)(t0 * p.HI));
                } else {
                    for (int c = 0; c < kchunks; ++c)
                        tma_load_2d(sB + (size_t)c * BN * 128, &tm_q, qfull, c * 64, (int)(t0 * p.HI));
                }
                int64_t t1;
                int n1;
                if (group_of(gi + 1, &t1, &n1))   // the next group's q^I into L2 while this group computes
                    for (int c = 0; c < (p.fp4 ? 1 : kchunks); ++c) tma_prefetch_2d(&tm_q, c * 64, (int)(t1 * p.HI));
            }
            if (p.fp4) {   // the group's q^I scales: lane r writes row r = the scale words of rows r + 32 j
                uint32_t wq[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int64_t row = t0 * p.HI + lane + 32 * j;   // (query, head) row of q^I
                    wq[j] = lane + 32 * j < p.bn && row < p.S * p.HI ? *reinterpret_cast<const uint32_t *>(p.qs + row * 4) : 0u;
                }
                *reinterpret_cast<uint4 *>(sSFB + (gi & 1) * 512 + lane * 16) = make_uint4(wq[0], wq[1], wq[2], wq[3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(qfull);
            }
            __syncwarp();
            ngr = gi + 1;
            for (int i = 0; i < ntiles; ++i, ++tile) {
                const int st = tile % p.stages;
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[st], ((tile / p.stages) & 1) ^ 1, abort, p.status))) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    mbar_arrive_expect_tx(&full[st], a_bytes);
                    if (p.fp4) {
                        tma_load_2d(sA + (size_t)st * a_bytes, &tm_k, &full[st], 0, i * BM);
                    } else {
                        for (int c = 0; c < kchunks; ++c)
                            tma_load_2d(sA + (size_t)st * a_bytes + (size_t)c * BM * 128, &tm_k, &full[st], c * 64, i * BM);
                    }
                }
                __syncwarp();
                issued = tile + 1;
            }
        }
        // never leave with copies in flight into this CTA's shared memory
        if (ngr > 0) mbar_wait(qfull, (uint32_t)((ngr - 1) & 1), abort, p.status, 100000000ull);
        for (int i = max(0, issued - p.stages); i < issued; ++i)
            mbar_wait(&full[i % p.stages], (i / p.stages) & 1, abort, p.status, 100000000ull);
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        const uint32_t idesc = idesc_bf16(BM, BN);
        const uint32_t idf0 = idesc_mxf4(BM, p.bn, 0), idf2 = idesc_mxf4(BM, p.bn, 2);
        int tile = 0;
        bool ok = true;
        int64_t t0;
        int ntiles;
        for (int64_t gi = 0; ok && group_of(gi, &t0, &ntiles); ++gi) {
            if (!__all_sync(0xffffffffu, mbar_wait(qfull, (uint32_t)(gi & 1), abort, p.status))) break;
            const uint32_t sfb = tmem_base + F4_SFB_COL + (uint32_t)(gi & 1) * 4;
            if (p.fp4) {   // the group's q^I scales into TMEM (ordered before this thread's later MMAs)
                tc_fence_after();
                if (elect_one()) tmem_cp_32x128b_x4(sfb, sdesc_plain(smem_u32(sSFB + (gi & 1) * 512), 16, 128));
                __syncwarp();
            }
            for (int i = 0; i < ntiles; ++i, ++tile) {
                const int st = tile % p.stages, buf = tile & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&tempty[buf], ((tile >> 1) & 1) ^ 1, abort, p.status)) ||
                    !__all_sync(0xffffffffu, mbar_wait(&full[st], (tile / p.stages) & 1, abort, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (p.fp4) {
                    if (elect_one()) {
                        const uint32_t sfa = tmem_base + F4_SFA_COL + (uint32_t)buf * 4;
                        tmem_cp_32x128b_x4(sfa, sdesc_plain(smem_u32(sSFA + i * 512), 16, 128));
                        const uint32_t a0 = smem_u32(sA + (size_t)st * a_bytes), b0 = smem_u32(sB);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks)   // channels 64 ks .. +63: scale bytes 2 ks, 2 ks + 1
                            mma_mxf4(tmem_base + buf * p.bn, sdesc_sw64(a0 + ks * 32, 512), sdesc_sw64(b0 + ks * 32, 512),
                                     ks ? idf2 : idf0, sfa | ((uint32_t)(2 * ks) << 30), sfb | ((uint32_t)(2 * ks) << 30),
                                     ks != 0);
                        mma_commit(&empty[st]);
                        mma_commit(&tfull[buf]);
                    }
                    __syncwarp();
                    continue;
                }
                if (elect_one()) {
                    const uint32_t a0 = smem_u32(sA + (size_t)st * a_bytes), b0 = smem_u32(sB);
                    for (int c = 0; c < kchunks; ++c) {
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint64_t ad = sdesc_sw128(a0 + c * BM * 128 + ks * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(b0 + c * BN * 128 + ks * 32, 16, 1024);
                            mma_bf16(tmem_base + buf * BN, ad, bd, idesc, (c | ks) != 0);
                        }
                    }
                    mma_commit(&empty[st]);
                    mma_commit(&tfull[buf]);
                }
                __syncwarp();
            }
            if (!ok) break;
            if (elect_one()) mma_commit(qempty);   // q^I is free once this group's MMAs complete
            __syncwarp();
        }
        // every MMA issued must be complete before TMEM is released: the last accumulator's commit
        // arrives once it and every earlier MMA have completed
        if (tile > 0) mbar_wait(&tfull[(tile - 1) & 1], ((tile - 1) >> 1) & 1, abort, p.status, 100000000ull);
    } else if (warp < 2 + EPI_THREADS / 32) {
        // ---------------- epilogue: scores into shared memory ----------------
        // warp w reads TMEM lane quarter w % 4 (entries 32*(w%4) .. +31 of the tile); warps 2-5 take
        // the first half of the group's queries, warps 6-9 the second half
        const int quarter = warp & 3;
        const int qhalf = (warp - 2) >> 2;
        const int qlo = qhalf * (p.Q >> 1), qhi = qlo + (p.Q >> 1);   // Q = 256 / HI is even
        const int etid = threadIdx.x - 64;
        int tile = 0;
        bool ok = true;
        int64_t t0;
        int ntiles;
        const int ct = p.chunk / BM;   // tiles per chunk
        int64_t unit = 0;              // (group, chunk) units so far: the scores buffers go round by unit
        float *scores = scores_all;
        int sb = 0;
        for (int64_t gi = 0; ok && group_of(gi, &t0, &ntiles); ++gi) {
            named_barrier_sync(1, EPI_THREADS);   // every epilogue thread is done with the previous weights
            for (int i = etid; i < p.Q * p.HI; i += EPI_THREADS) {
                const int64_t t = t0 + i / p.HI;
                sw[i] = t < p.S ? p.w[t * p.HI + (i % p.HI)] : 0.f;
            }
            named_barrier_sync(1, EPI_THREADS);
            if (ntiles == 0) {   // nothing visible to the group yet: one empty chunk, so its rows get -1
                sb = (int)(unit % p.nsb);
                const int64_t use = unit / p.nsb;
                if (use > 0 &&
                    !__all_sync(0xffffffffu, mbar_wait(&sempty[sb], (uint32_t)((use - 1) & 1), abort, p.status))) {
                    ok = false;
                    break;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sfull[sb]);
                ++unit;
            }
            for (int i = 0; i < ntiles; ++i, ++tile) {
                if (i % ct == 0) {   // a new chunk: its scores buffer once the top-k is done with it
                    sb = (int)(unit % p.nsb);
                    const int64_t use = unit / p.nsb;   // earlier uses of this scores buffer
                    if (use > 0 &&
                        !__all_sync(0xffffffffu, mbar_wait(&sempty[sb], (uint32_t)((use - 1) & 1), abort, p.status))) {
                        ok = false;
                        break;
                    }
                    scores = scores_all + (size_t)sb * p.Q * p.qstride + p.kcap;
                }
                const int buf = tile & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (tile >> 1) & 1, abort, p.status))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int s = (i % ct) * BM + quarter * 32 + lane;   // entry within the chunk
                const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) + buf * p.bn;
                for (int q = qlo; q < qhi; ++q) {
                    // four independent partial sums break the dependent multiply-add chain
                    float acc4[4] = {0.f, 0.f, 0.f, 0.f};
                    // columns [q*HI, (q+1)*HI) of this buffer; never read past them (HI = 16 uses x16 loads)
                    for (int h0 = 0; h0 < p.HI; h0 += 16) {
                        const float4 *wq4 = reinterpret_cast<const float4 *>(sw + q * p.HI + h0);
                        if (h0 + 32 <= p.HI) {
                            float v[32];
                            tmem_ld32(taddr + q * p.HI + h0, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 w4 = wq4[j];
                                acc4[0] = fmaf(w4.x, fmaxf(v[4 * j], 0.f), acc4[0]);
                                acc4[1] = fmaf(w4.y, fmaxf(v[4 * j + 1], 0.f), acc4[1]);
                                acc4[2] = fmaf(w4.z, fmaxf(v[4 * j + 2], 0.f), acc4[2]);
                                acc4[3] = fmaf(w4.w, fmaxf(v[4 * j + 3], 0.f), acc4[3]);
                            }
                            h0 += 16;
                        } else {
                            float v[16];
                            tmem_ld16(taddr + q * p.HI + h0, v);
                            tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const float4 w4 = wq4[j];
                                acc4[0] = fmaf(w4.x, fmaxf(v[4 * j], 0.f), acc4[0]);
                                acc4[1] = fmaf(w4.y, fmaxf(v[4 * j + 1], 0.f), acc4[1]);
                                acc4[2] = fmaf(w4.z, fmaxf(v[4 * j + 2], 0.f), acc4[2]);
                                acc4[3] = fmaf(w4.w, fmaxf(v[4 * j + 3], 0.f), acc4[3]);
                            }
                        }
                    }
                    const float acc = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
                    scores[q * p.qstride + s] = acc + 0.0f;
                }
                tc_fence_before();
                mbar_arrive(&tempty[buf]);
                if (i % ct == ct - 1 || i + 1 == ntiles) {   // this warp's scores of the chunk are in place
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sfull[sb]);
                    ++unit;
                }
            }
            if (!ok) break;
        }
    } else {
        // ---------------- exact top-k of the previous group's queries, one query per pair of warps ----
        const int pair = (warp - 2 - EPI_THREADS / 32) >> 1;
        const int pt = threadIdx.x & 63;
        const int bar = 2 + pair;
        uint32_t *scratch = hist + pair * (PBINS + 80);
        int32_t *sel = sel_all + pair * p.kcap;
        const int ct = p.chunk / BM;
        int64_t unit = 0;
        int64_t t0;
        int ntiles;
        bool ok = true;
        for (int64_t gi = 0; ok && group_of(gi, &t0, &ntiles); ++gi) {
            const int nch = max(1, (ntiles + ct - 1) / ct);   // a group with no entries yet: one empty chunk
            for (int c = 0; c < nch; ++c, ++unit) {
                const int sb = (int)(unit % p.nsb);
                if (!__all_sync(0xffffffffu, mbar_wait(&sfull[sb], (uint32_t)((unit / p.nsb) & 1), abort, p.status))) {
                    ok = false;
                    break;
                }
                float *scores = scores_all + (size_t)sb * p.Q * p.qstride;
                for (int q = pair; q < p.Q; q += 4) {
                    const int64_t t = t0 + q;
                    if (t >= p.S) continue;
                    const int n = (int)visible_entries(p.pos0 + t, p.m, p.T);
                    int32_t *orow = p.idx + t * (int64_t)p.k;
                    float *sq = scores + (size_t)q * p.qstride + p.kcap;   // the chunk's scores of query q
                    if (p.kcap == 0) {   // every entry in one chunk: rank it in place
                        if (n > p.k && n <= 2048)
                            topk_pair_reg(sq, n, p.k, scratch, bar, orow);
                        else
                            topk_pair(sq, n, p.k, scratch, bar, orow);
                        continue;
                    }
                    const int nc = min(max(n - c * p.chunk, 0), p.chunk);   // this query's entries in the chunk
                    if (nc == 0) {
                        if (c == 0)   // nothing visible yet: every slot is -1
                            for (int j = pt; j < p.k; j += 64) orow[j] = -1;
                        continue;
                    }
                    const int r = c == 0 ? 0 : run_cnt[q];
                    for (int j = pt; j < r; j += 64) sq[j - r] = run_sc[q * p.kcap + j];   // running set first
                    pair_sync(bar);
                    const int nn = r + nc;
                    if (nn > p.k && nn <= 2048)
                        topk_pair_reg(sq - r, nn, p.k, scratch, bar, sel);
                    else
                        topk_pair(sq - r, nn, p.k, scratch, bar, sel);
                    // the new running set: positions below r are running entries, the rest chunk entries. Its
                    // scores are read from the ranked buffer (the running scores were copied there), its
                    // entry indices replace the positions in `sel` (each slot by its own thread), then move.
                    const int r2 = min(p.k, nn);
                    for (int j = pt; j < r2; j += 64) {
                        const int pos = sel[j];
                        run_sc[q * p.kcap + j] = sq[pos - r];
                        sel[j] = pos < r ? run_idx[q * p.kcap + pos] : c * p.chunk + (pos - r);
                    }
                    pair_sync(bar);
                    for (int j = pt; j < r2; j += 64) run_idx[q * p.kcap + j] = sel[j];
                    if (pt == 0) run_cnt[q] = r2;
                    pair_sync(bar);
                    if ((c + 1) * p.chunk >= n)   // the query's last chunk: its selection, ascending
                        for (int j = pt; j < p.k; j += 64) orow[j] = j < r2 ? run_idx[q * p.kcap + j] : -1;
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[sb]);   // the buffer may take a later chunk's scores
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// ---- host: tensor maps ------------------------------------------------------------------------------

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (fn == nullptr) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

static bool make_tmap_sw128(CUtensorMap *map, const void *base, CUtensorMapDataType dt, uint32_t esize, uint64_t rows,
                            uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esize};
    cuuint32_t box[2] = {128 / esize, box_rows};   // one 128-byte swizzle span per box row
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// 2-D bf16 tensor map over a row-major [rows, cols] matrix, box [box_rows, 64], 128-byte swizzle.
bool make_tmap_bf16_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    return make_tmap_sw128(map, base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, rows, cols, box_rows);
}

// 2-D fp32 tensor map over a row-major [rows, cols] matrix, box [box_rows, 32], 128-byte swizzle.
bool make_tmap_f32_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    return make_tmap_sw128(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, rows, cols, box_rows);
}

bool make_tmap_u8_rows(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr || cols % 16 != 0 || cols > 256) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D byte tensor map over [rows, 64] (64-byte rows), box [box_rows, 64], 64-byte swizzle: the K-major
// layout of packed FP4 operands with 128 channels per row.
bool make_tmap_u8_sw64(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {64, rows};
    cuuint64_t strides[1] = {64};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Shared-memory plan of the fused indexer: every entry in one chunk when the scores of a group's
// queries fit (two scores buffers when three key stages still fit), else (bf16, k <= 1024) chunks of
// entries with a running top-k per query, one scores buffer, the chunk as long as shared memory allows.
struct IdxPlan {
    int bn, Q, T_cap, nsb, stages, chunk, kcap, qstride;
    size_t smem;
};

static bool plan_index_topk(int64_t T, int HI, int dI, int k, bool fp4, IdxPlan *pl)
{
    if (T < 1 || T > (1ll << 24) || !(dI == 64 || dI == 128) || !(HI == 16 || HI == 32 || HI == 64 || HI == 128))
        return false;
    if (fp4 && (dI != 128 || HI > 64 || T > 4096)) return false;
    pl->bn = fp4 ? 128 : BN;   // MXFP4: two 128-column accumulators leave TMEM room for the scales
    pl->Q = pl->bn / HI;
    pl->T_cap = (int)((T + BM - 1) / BM * BM);
    const size_t a_bytes = fp4 ? (size_t)BM * 64 : (size_t)(dI / 64) * BM * 128;
    const size_t b_bytes = fp4 ? (size_t)pl->bn * 64 : (size_t)(dI / 64) * BN * 128;
    const size_t sf_bytes = fp4 ? (size_t)(pl->T_cap / BM) * 512 + 1024 : 0;
    const size_t budget = 227 * 1024;
    auto fixed_of = [&](int nsb, int qstride, int kcap) {
        const size_t run = kcap > 0 ? (size_t)pl->Q * kcap * 8 + (size_t)(pl->Q + 3) / 4 * 16 + 4 * (size_t)kcap * 4 : 0;
        return 1024 + b_bytes + (size_t)nsb * pl->Q * qstride * 4 + BN * 4 + 4 * (PBINS + 80) * 4 + run + sf_bytes + 256;
    };
    pl->kcap = 0;
    pl->chunk = pl->qstride = pl->T_cap;
    for (pl->nsb = 2; pl->nsb >= 1; --pl->nsb)
        if (fixed_of(pl->nsb, pl->qstride, 0) + 2 * a_bytes <= budget) break;
    if (pl->nsb < 1) {   // chunks of entries with a running top-k
        if (fp4 || k > 1024) return false;
        pl->nsb = 1;
        pl->kcap = (k + 3) & ~3;
        const size_t base = fixed_of(1, 0, pl->kcap) + 2 * a_bytes;
        if (base >= budget) return false;
        const int64_t room = (int64_t)((budget - base) / ((size_t)pl->Q * 4)) - pl->kcap;   // floats per query
        pl->chunk = (int)std::min<int64_t>(room / BM * BM, pl->T_cap);
        if (pl->chunk < 4 * BM) return false;
        pl->qstride = pl->kcap + pl->chunk;
    }
    const size_t fixed = fixed_of(pl->nsb, pl->qstride, pl->kcap);
    pl->stages = (int)std::min<size_t>(fp4 ? 8 : 4, (budget - fixed) / a_bytes);
    if (pl->stages < 2) return false;
    pl->smem = fixed + (size_t)pl->stages * a_bytes;
    return true;
}

// Launch of the fused indexer for either operand format.
static cudaError_t launch_index_topk(const void *qI, const void *kI, const uint8_t *qs, const uint8_t *ks, bool fp4,
                                     const float *w, int64_t S, int64_t pos0, int64_t T, int HI, int dI, int m, int k,
                                     int32_t *idx, int32_t *status, cudaStream_t stream)
{
    if (S == 0) return cudaSuccess;
    IdxPlan pl;
    if (!plan_index_topk(T, HI, dI, k, fp4, &pl)) return cudaErrorInvalidValue;
    IdxParams p;
    p.w = w;
    p.idx = idx;
    p.status = status;
    p.S = S;
    p.pos0 = pos0;
    p.T = T;
    p.HI = HI;
    p.dI = dI;
    p.m = m;
    p.k = k;
    p.fp4 = fp4 ? 1 : 0;
    p.qs = qs;
    p.ks = ks;
    p.bn = pl.bn;
    p.Q = pl.Q;
    p.T_cap = pl.T_cap;
    p.nsb = pl.nsb;
    p.stages = pl.stages;
    p.chunk = pl.chunk;
    p.kcap = pl.kcap;
    p.qstride = pl.qstride;
    p.ngroups = (S + p.Q - 1) / p.Q;
    CUtensorMap tq, tk;
    if (fp4) {
        if (!make_tmap_u8_sw64(&tq, qI, (uint64_t)S * HI, (uint32_t)p.bn)) return cudaErrorInvalidValue;
        if (!make_tmap_u8_sw64(&tk, kI, (uint64_t)T, BM)) return cudaErrorInvalidValue;
    } else {
        if (!make_tmap_bf16_sw128(&tq, qI, (uint64_t)S * HI, dI, BN)) return cudaErrorInvalidValue;
        if (!make_tmap_bf16_sw128(&tk, kI, (uint64_t)T, dI, BM)) return cudaErrorInvalidValue;
    }
    cudaError_t e = ensure_smem_limit(reinterpret_cast<const void *>(index_topk_tc_kernel), pl.smem);
    if (e != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if ((e = current_device_sms(&dev, &nsm)) != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<int64_t>(nsm, p.ngroups);   // persistent
    index_topk_tc_kernel<<<grid, NUM_THREADS, pl.smem, stream>>>(tq, tk, p);
    return cudaGetLastError();
}

bool index_topk_tc_supported(int64_t T, int HI, int dI, int k)
{
    IdxPlan pl;
    return encode_fn() != nullptr && plan_index_topk(T, HI, dI, k, false, &pl);
}

cudaError_t launch_index_topk_tc(const uint16_t *qI, const uint16_t *kI, const float *w, int64_t S, int64_t pos0,
                                 int64_t T, int HI, int dI, int m, int k, int32_t *idx, int32_t *status,
                                 cudaStream_t stream)
{
    return launch_index_topk(qI, kI, nullptr, nullptr, false, w, S, pos0, T, HI, dI, m, k, idx, status, stream);
}

bool index_topk_fp4_supported(int64_t T, int HI, int dI, int k)
{
    IdxPlan pl;
    return encode_fn() != nullptr && plan_index_topk(T, HI, dI, k, true, &pl);
}

cudaError_t launch_index_topk_fp4(const uint8_t *qc, const uint8_t *qs, const float *w, const uint8_t *kc,
                                  const uint8_t *ks, int64_t S, int64_t pos0, int64_t T, int HI, int dI, int m, int k,
                                  int32_t *idx, int32_t *status, cudaStream_t stream)
{
    return launch_index_topk(qc, kc, qs, ks, true, w, S, pos0, T, HI, dI, m, k, idx, status, stream);
}

}  // namespace csa
