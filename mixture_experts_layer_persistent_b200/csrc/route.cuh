// route.cuh -- router weight split, scoring and top-k selection, and the
// deterministic counting sort that turns the selection into per-expert row
// ranges (counts, prefix offsets, stable permutation, row maps).
//
// Selection rule (DeepSeek-V3-type layer, "Cursor åpner megakernelen…", last
// paragraph): softmax scoring selects the k largest logits; sigmoid scoring
// selects on s + e_bias after keeping the topk_group groups with the largest
// sum of their two best biased scores.  Every comparison orders (score
// descending, index ascending), so ties go to the lower expert / group index.
// Weights: softmax over the selected logits, or the unbiased sigmoid scores
// divided by their sum; both times routed_scale.
#pragma once
#include "ptx.cuh"

namespace mok {

// Router weights as three bf16 terms: Wr = hi + mid + lo to within 2^-25
// relative, laid out [E, 3H] = [hi | mid | lo] along K, so that the tensor-core
// contraction of x (bf16, exact) with the three terms reproduces the fp32
// router logits.  Each difference below is exact in fp32.
// It also writes the one-group row range {0, T} the router contraction reads.
__device__ __forceinline__ void router_split_elem(long long i, const float *__restrict__ Wr,
                                                  __nv_bfloat16 *__restrict__ Wr3, int H)
{
    const int e = (int)(i / H), h = (int)(i % H);
    const float w = Wr[i];
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    __nv_bfloat16 *row = Wr3 + (size_t)e * 3 * H;
    row[h] = hi;
    row[H + h] = mid;
    row[2 * H + h] = lo;
}

__global__ void __launch_bounds__(256) router_split_kernel(const float *__restrict__ Wr,
                                                           __nv_bfloat16 *__restrict__ Wr3, int E, int H,
                                                           int *__restrict__ all_rows, int T)
{
    griddep_enter();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) {
        all_rows[0] = 0;
        all_rows[1] = T;
    }
    if (i < (long long)E * H) router_split_elem(i, Wr, Wr3, H);
}

struct SelectArgs {
    const float *partial;       // [n_split, T, 256] partial logits (tensor-core K splits)
    int n_split;
    const float *e_bias;        // [E] or null
    const float *logit_bias;    // [E] or null
    int T, E, k;
    int score_fn, n_group, topk_group;
    float routed_scale;
    int *topk_idx;              // [T, k]
    float *topk_w;              // [T, k]
    float *topk_p;              // [T, k] sigmoid score s (sigmoid) or w / routed_scale (softmax)
    int *hist;                  // null, or [chunks of kDispatchChunk tokens, E] counts, zero
                                // before: the selection also counts each (token, slot) there
};

// tokens per dispatch chunk: enough chunks that the placement spreads over many
// CTAs, few enough mask words per expert (kDispatchChunk / 32) for the rank scan
constexpr int kDispatchChunk = 256;
constexpr int kMaxRouterSplits = 8;     // K splits of the router GEMM at most
constexpr int kMaskWords = kDispatchChunk / 32;

// one (value, index) candidate; larger value wins, then lower index
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib)
{
    return va > vb || (va == vb && ia < ib);
}

__device__ __forceinline__ void warp_argmax(float &v, int &i)
{
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, d);
        const int oi = __shfl_xor_sync(0xffffffffu, i, d);
        if (better(ov, oi, v, i)) {
            v = ov;
            i = oi;
        }
    }
}

// A selection score that is NaN (a non-finite activation or bias) ranks below
// every other score, as -inf does; the selection below still returns k distinct
// experts in [0, E), ties going to the lower index.
__device__ __forceinline__ float rank_score(float v) { return v == v ? v : -INFINITY; }

// Selection of one token by one warp.  Lane l holds experts l + 32 i.  The
// logit is the sum of the K-split partials in split order plus logit_bias;
// selection as above.  row: 256 floats of shared memory owned by the warp.
__device__ __forceinline__ void select_token(const SelectArgs &a, int t, int lane, float *row)
{
    const int E = a.E;
    const int npl = (E + 31) / 32;
    // every partial and bias of the token is loaded before the first sum (one
    // round trip instead of one per split and expert); the sums keep split order
    float part[kMaxRouterSplits][8], lb[8], eb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        const bool on = i < npl && e < E;
#pragma unroll
        for (int s = 0; s < kMaxRouterSplits; ++s)
            part[s][i] = on && s < a.n_split ? a.partial[((size_t)s * a.T + t) * 256 + e] : 0.0f;
        lb[i] = on && a.logit_bias ? a.logit_bias[e] : 0.0f;
        eb[i] = on && a.e_bias ? a.e_bias[e] : 0.0f;
    }
    float lgv[8], sel[8], sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        lgv[i] = 0.0f;
        sel[i] = -INFINITY;
        sc[i] = 0.0f;
        if (i < npl && e < E) {
            float lg = 0.0f;
#pragma unroll
            for (int s = 0; s < kMaxRouterSplits; ++s)
                if (s < a.n_split) lg += part[s][i];
            if (a.logit_bias) lg += lb[i];
            lgv[i] = lg;
            if (a.score_fn == 0) {
                sel[i] = rank_score(lg);
            } else {
                const float sg = 1.0f / (1.0f + expf(-lg));
                sc[i] = sg;
                sel[i] = rank_score(sg + (a.e_bias ? eb[i] : 0.0f));
            }
        }
    }
    if (a.n_group > 1 && a.topk_group < a.n_group) {
        // group score: sum of the two best selection scores of the group
        const int gs = E / a.n_group;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (i < npl && e < E) row[e] = sel[i];
        }
        __syncwarp();
        float gsc = -INFINITY;
        if (lane < a.n_group) {
            float b1 = -INFINITY, b2 = -INFINITY;
            for (int m = 0; m < gs; ++m) {
                const float v = row[lane * gs + m];
                if (v > b1) { b2 = b1; b1 = v; }
                else if (v > b2) { b2 = v; }
            }
            gsc = rank_score(gs > 1 ? b1 + b2 : b1);
        }
        unsigned keep = 0;   // bit g set: group g kept
        for (int r = 0; r < a.topk_group; ++r) {
            // groups already kept and lanes past the last group never win, so the
            // topk_group kept groups are distinct even when their scores are -inf
            const bool cand = lane < a.n_group && !(keep & (1u << lane));
            float v = cand ? gsc : -INFINITY;
            int gi = cand ? lane : 1 << 30;
            warp_argmax(v, gi);
            if (gi < a.n_group) keep |= 1u << gi;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (i < npl && e < E && !(keep & (1u << (e / gs)))) sel[i] = -INFINITY;
        }
    }
    // top-k by repeated warp argmax over the experts not yet taken; k <= E, so
    // every round finds a candidate and bi is always an expert index below E
    // lane j < k keeps the j-th selected expert and its value (k <= 16)
    int my_idx = 0;
    float my_val = 0.0f;
    unsigned taken = 0;      // bit i: expert lane + 32 i already selected
    for (int j = 0; j < a.k; ++j) {
        float bv = -INFINITY;
        int bi = 1 << 30;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (i < npl && e < E && !(taken & (1u << i)) && better(sel[i], e, bv, bi)) {
                bv = sel[i];
                bi = e;
            }
        }
        warp_argmax(bv, bi);
        float wv = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (lane + 32 * i == bi) {
                taken |= 1u << i;                                     // the owner retires the winner
                wv = a.score_fn == 0 ? lgv[i] : sc[i];               // logit (softmax) or sigmoid score
            }
        const float val = __shfl_sync(0xffffffffu, wv, bi & 31);
        if (lane == j) {
            my_idx = bi;
            my_val = val;
        }
    }
    // renormalised weights: softmax over the selected logits (shifted by the
    // first, the largest) or the selected sigmoid scores; the sum runs in
    // selection order
    float p = 0.0f;
    if (a.score_fn == 0) {
        const float m = __shfl_sync(0xffffffffu, my_val, 0);
        if (lane < a.k) p = expf(my_val - m);
    } else if (lane < a.k) {
        p = my_val;
    }
    float wsum = 0.0f;
    for (int j = 0; j < a.k; ++j) wsum += __shfl_sync(0xffffffffu, p, j);
    if (lane < a.k) {
        const float q = p / wsum;
        const size_t o = (size_t)t * a.k + lane;
        a.topk_idx[o] = my_idx;
        a.topk_w[o] = a.routed_scale * q;
        a.topk_p[o] = a.score_fn == 0 ? q : my_val;
        if (a.hist) atomicAdd(&a.hist[(size_t)(t / kDispatchChunk) * E + my_idx], 1);
    }
}

// One warp per token.
__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a)
{
    griddep_enter();
    __shared__ float s_row[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= a.T) return;
    select_token(a, t, lane, s_row[warp]);
}

// ------------------------------------------------------------------ dispatch
struct DispatchArgs {
    const int *topk_idx;   // [T, k]
    const float *topk_w;   // [T, k]
    int T, k, E, S;
    int chunk_rows;        // row chunk of the router-gradient partial sums
    int *hist;             // [C, E] (tokens of chunk c choosing e), then the chunk's base row
    int *counts;           // [E]
    int *offsets;          // [E + S + 1] sorted-row ranges (routed, then shared)
    int *gorder;           // [E + S] groups by rows descending, index ascending
    int *chunk_start;      // [E + 1] prefix of ceil(counts / chunk_rows)
    int *perm;             // [T k]
    int *inv_perm;         // [T k]
    int *row_token;        // [R]
    int *row_slot;         // [R]
    float *row_w;          // [R]
    int *status;           // device status word
};

// A routing index outside [0, E) cannot come out of the selection above; if one
// is ever met, it is counted and placed as expert 0 (both dispatch kernels map
// it the same way, so every row range stays consistent and in bounds) and the
// status word records MOK_STATUS_BAD_INDEX.
__device__ __forceinline__ int checked_expert(int e, int E, int *status)
{
    if (static_cast<unsigned>(e) < static_cast<unsigned>(E)) return e;
    atomicOr(status, kStatusBadIndex);
    return 0;
}

// Integer counting sort of the T*k (token, slot) pairs by expert, stable in
// token order, in three launches: per-chunk histograms, a per-expert scan over
// chunks and experts, and per-chunk placement.  Every count is an integer, so
// the result is the same whatever the order of the atomics.
__global__ void __launch_bounds__(1024) dispatch_count_kernel(const DispatchArgs a)
{
    griddep_enter();
    __shared__ int s_cnt[256];
    const int c = blockIdx.x, tid = threadIdx.x;
    for (int e = tid; e < a.E; e += blockDim.x) s_cnt[e] = 0;
    __syncthreads();
    const int t = c * kDispatchChunk + tid;
    if (t < a.T)
        for (int j = 0; j < a.k; ++j) atomicAdd(&s_cnt[checked_expert(a.topk_idx[(size_t)t * a.k + j], a.E, a.status)], 1);
    __syncthreads();
    for (int e = tid; e < a.E; e += blockDim.x) a.hist[(size_t)c * a.E + e] = s_cnt[e];
}

// One block: counts, exclusive offsets, each chunk's first row per expert (in
// place of its histogram), router-gradient chunk starts and the group order.
__global__ void __launch_bounds__(256) dispatch_scan_kernel(const DispatchArgs a, int n_chunks)
{
    griddep_enter();
    __shared__ int s_cnt[256];
    __shared__ int s_off[257];
    const int e = threadIdx.x, E = a.E, T = a.T;
    int total = 0;
    if (e < E) {
#pragma unroll 8
        for (int c = 0; c < n_chunks; ++c) total += a.hist[(size_t)c * E + e];
    }
    s_cnt[e] = e < E ? total : 0;
    __syncthreads();
    if (e == 0) {
        int acc = 0, cacc = 0;
        for (int q = 0; q < E; ++q) {
            s_off[q] = acc;
            a.counts[q] = s_cnt[q];
            a.offsets[q] = acc;
            a.chunk_start[q] = cacc;
            acc += s_cnt[q];
            cacc += (s_cnt[q] + a.chunk_rows - 1) / a.chunk_rows;
        }
        a.chunk_start[E] = cacc;
        for (int s = 0; s <= a.S; ++s) a.offsets[E + s] = acc + s * T;
    }
    __syncthreads();
    if (e < E) {
        int run = s_off[e];
        for (int c = 0; c < n_chunks; ++c) {
            const int h = a.hist[(size_t)c * E + e];
            a.hist[(size_t)c * E + e] = run;
            run += h;
        }
    }
    // group order: longest first, lower index on ties
    for (int g = e; g < E + a.S; g += 256) {
        const int cg = g < E ? s_cnt[g] : T;
        int rank = 0;
        for (int h = 0; h < E + a.S; ++h) {
            const int ch = h < E ? s_cnt[h] : T;
            rank += (ch > cg) || (ch == cg && h < g);
        }
        a.gorder[rank] = g;
    }
}

// The scan and the placement of one chunk in one CTA (any block size >= 256),
// for the persistent forward: every CTA that owns a chunk derives its own base
// rows from the per-chunk counts (exclusive offsets over experts plus the
// counts of the earlier chunks), so no grid-wide step sits between the scan
// and the placement; CTA `writer` also writes counts, offsets, the
// router-gradient chunk starts and the group order.  The placement is the one
// of dispatch_place_kernel below, with the token of a thread strided by the
// block size.  s_mask: [256][kMaskWords] words, s_base / s_cnt: 256 ints each.
__device__ __forceinline__ void dispatch_scan_place_chunk(const DispatchArgs &a, int c, int n_chunks, bool writer,
                                                          uint32_t (*s_mask)[kMaskWords], int *s_base, int *s_cnt)
{
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int E = a.E, k = a.k, kk = a.k + a.S, T = a.T;
    for (int q = tid; q < E * kMaskWords; q += nthr) (&s_mask[0][0])[q] = 0u;
    if (tid < E) {
        int total = 0, before = 0;
#pragma unroll 8
        for (int cc = 0; cc < n_chunks; ++cc) {
            const int h = a.hist[(size_t)cc * E + tid];
            if (cc < c) before += h;
            total += h;
        }
        s_cnt[tid] = total;
        s_base[tid] = before;
    }
    __syncthreads();
    if (tid == 0) {
        int acc = 0, cacc = 0;
        for (int q = 0; q < E; ++q) {
            const int cnt = s_cnt[q];
            s_base[q] += acc;
            if (writer) {
                a.counts[q] = cnt;
                a.offsets[q] = acc;
                a.chunk_start[q] = cacc;
            }
            acc += cnt;
            cacc += (cnt + a.chunk_rows - 1) / a.chunk_rows;
        }
        if (writer) {
            a.chunk_start[E] = cacc;
            for (int s2 = 0; s2 <= a.S; ++s2) a.offsets[E + s2] = acc + s2 * T;
        }
    }
    if (writer) {
        for (int g = tid; g < E + a.S; g += nthr) {
            const int cg = g < E ? s_cnt[g] : T;
            int rank = 0;
            for (int h = 0; h < E + a.S; ++h) {
                const int ch = h < E ? s_cnt[h] : T;
                rank += (ch > cg) || (ch == cg && h < g);
            }
            a.gorder[rank] = g;
        }
    }
    __syncthreads();
    const int t0 = c * kDispatchChunk;
    const int nt = min(kDispatchChunk, T - t0);
    for (int l = tid; l < nt; l += nthr)
        for (int j = 0; j < k; ++j)
            atomicOr(&s_mask[checked_expert(a.topk_idx[(size_t)(t0 + l) * k + j], E, a.status)][l >> 5], 1u << (l & 31));
    __syncthreads();
    for (int l = tid; l < nt; l += nthr) {
        const int t = t0 + l, word = l >> 5, bit = l & 31;
        for (int j = 0; j < k; ++j) {
            const int e = checked_expert(a.topk_idx[(size_t)t * k + j], E, a.status);
            int rank = __popc(s_mask[e][word] & ((1u << bit) - 1u));
            for (int w = 0; w < word; ++w) rank += __popc(s_mask[e][w]);
            const int pos = s_base[e] + rank;
            const int sl = t * k + j;
            a.perm[pos] = sl;
            a.inv_perm[sl] = pos;
            a.row_token[pos] = t;
            a.row_slot[pos] = t * kk + j;
            a.row_w[pos] = a.topk_w[sl];
        }
        const long long TK = (long long)T * k;
        for (int s2 = 0; s2 < a.S; ++s2) {
            const long long pos = TK + (long long)s2 * T + t;
            a.row_token[pos] = t;
            a.row_slot[pos] = t * kk + k + s2;
            a.row_w[pos] = 1.0f;
        }
    }
    __syncthreads();
}

// Per chunk: per-expert token bitmasks give each (token, slot) its rank among
// the chunk's earlier tokens of that expert; row = chunk base + rank.
__global__ void __launch_bounds__(1024) dispatch_place_kernel(const DispatchArgs a)
{
    griddep_enter();
    __shared__ uint32_t s_mask[256][kMaskWords];
    const int c = blockIdx.x, tid = threadIdx.x;
    const int E = a.E, k = a.k, kk = a.k + a.S, T = a.T;
    for (int q = tid; q < E * kMaskWords; q += blockDim.x) (&s_mask[0][0])[q] = 0u;
    __syncthreads();
    const int t = c * kDispatchChunk + tid;
    const int word = tid >> 5, bit = tid & 31;
    if (t < T)
        for (int j = 0; j < k; ++j) atomicOr(&s_mask[checked_expert(a.topk_idx[(size_t)t * k + j], E, a.status)][word], 1u << bit);
    __syncthreads();
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = checked_expert(a.topk_idx[(size_t)t * k + j], E, a.status);
            int rank = __popc(s_mask[e][word] & ((1u << bit) - 1u));
            for (int w = 0; w < word; ++w) rank += __popc(s_mask[e][w]);
            const int pos = a.hist[(size_t)c * E + e] + rank;
            const int sl = t * k + j;
            a.perm[pos] = sl;
            a.inv_perm[sl] = pos;
            a.row_token[pos] = t;
            a.row_slot[pos] = t * kk + j;
            a.row_w[pos] = a.topk_w[sl];
        }
        // shared experts: every token, in token order, weight 1
        const long long TK = (long long)T * k;
        for (int s = 0; s < a.S; ++s) {
            const long long pos = TK + (long long)s * T + t;
            a.row_token[pos] = t;
            a.row_slot[pos] = t * kk + k + s;
            a.row_w[pos] = 1.0f;
        }
    }
}

}  // namespace mok
