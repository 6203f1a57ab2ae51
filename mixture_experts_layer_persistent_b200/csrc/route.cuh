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
__global__ void __launch_bounds__(256) router_split_kernel(const float *__restrict__ Wr,
                                                           __nv_bfloat16 *__restrict__ Wr3, int E, int H,
                                                           int *__restrict__ all_rows, int T)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i == 0) {
        all_rows[0] = 0;
        all_rows[1] = T;
    }
    if (i >= (long long)E * H) return;
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
};

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

// One warp per token.  Lane l holds experts l + 32 i.  The logit is the sum of
// the K-split partials in split order plus logit_bias; selection as above.
__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a)
{
    __shared__ float s_row[8][256];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * 8 + warp;
    if (t >= a.T) return;
    const int E = a.E;
    const int npl = (E + 31) / 32;
    float *row = s_row[warp];
    float lgv[8], sel[8], sc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int e = lane + 32 * i;
        lgv[i] = 0.0f;
        sel[i] = -INFINITY;
        sc[i] = 0.0f;
        if (i < npl && e < E) {
            float lg = 0.0f;
            for (int s = 0; s < a.n_split; ++s) lg += a.partial[((size_t)s * a.T + t) * 256 + e];
            if (a.logit_bias) lg += a.logit_bias[e];
            lgv[i] = lg;
            if (a.score_fn == 0) {
                sel[i] = lg;
            } else {
                const float sg = 1.0f / (1.0f + expf(-lg));
                sc[i] = sg;
                sel[i] = sg + (a.e_bias ? a.e_bias[e] : 0.0f);
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
            gsc = gs > 1 ? b1 + b2 : b1;
        }
        unsigned keep = 0;   // bit g set: group g kept
        for (int r = 0; r < a.topk_group; ++r) {
            float v = lane < a.n_group ? gsc : -INFINITY;
            int gi = lane < a.n_group ? lane : 1 << 30;
            if (keep & (1u << (lane & 31))) v = -INFINITY;
            warp_argmax(v, gi);
            keep |= 1u << gi;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (i < npl && e < E && !(keep & (1u << (e / gs)))) sel[i] = -INFINITY;
        }
    }
    // top-k by repeated warp argmax
    int my_idx[16];
    float my_val[16];
    for (int j = 0; j < a.k; ++j) {
        float bv = -INFINITY;
        int bi = 1 << 30;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            if (i < npl && e < E && better(sel[i], e, bv, bi)) {
                bv = sel[i];
                bi = e;
            }
        }
        warp_argmax(bv, bi);
        my_idx[j] = bi;
        float wv = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (lane + 32 * i == bi) {
                sel[i] = -INFINITY;                                   // the owner retires the winner
                wv = a.score_fn == 0 ? lgv[i] : sc[i];               // logit (softmax) or sigmoid score
            }
        my_val[j] = __shfl_sync(0xffffffffu, wv, bi & 31);
    }
    if (lane == 0) {
        float wsum = 0.0f;
        float p[16];
        if (a.score_fn == 0) {
            const float m = my_val[0];
            for (int j = 0; j < a.k; ++j) { p[j] = expf(my_val[j] - m); wsum += p[j]; }
        } else {
            for (int j = 0; j < a.k; ++j) { p[j] = my_val[j]; wsum += p[j]; }
        }
        for (int j = 0; j < a.k; ++j) {
            const float q = p[j] / wsum;
            a.topk_idx[(size_t)t * a.k + j] = my_idx[j];
            a.topk_w[(size_t)t * a.k + j] = a.routed_scale * q;
            a.topk_p[(size_t)t * a.k + j] = a.score_fn == 0 ? q : my_val[j];
        }
    }
}

// ------------------------------------------------------------------ dispatch
struct DispatchArgs {
    const int *topk_idx;   // [T, k]
    const float *topk_w;   // [T, k]
    int T, k, E, S;
    int chunk_rows;        // row chunk of the router-gradient partial sums
    int *counts;           // [E]
    int *offsets;          // [E + S + 1] sorted-row ranges (routed, then shared)
    int *gorder;           // [E + S] groups by rows descending, index ascending
    int *chunk_start;      // [E + 1] prefix of ceil(counts / chunk_rows)
    int *perm;             // [T k]
    int *inv_perm;         // [T k]
    int *row_token;        // [R]
    int *row_slot;         // [R]
    float *row_w;          // [R]
};

// One block of 1024 threads: integer counting sort, bit-exact and stable in
// token order.  Chunks of 1024 tokens: per-expert token bitmasks give each
// (token, slot) its rank among earlier tokens of the chunk.
__global__ void __launch_bounds__(1024) dispatch_kernel(const DispatchArgs a)
{
    __shared__ int s_cnt[256];
    __shared__ int s_base[256];
    __shared__ uint32_t s_mask[256][32];
    const int tid = threadIdx.x;
    const int E = a.E, k = a.k, T = a.T, kk = a.k + a.S;
    const long long TK = (long long)T * k;
    for (int e = tid; e < E; e += 1024) s_cnt[e] = 0;
    __syncthreads();
    for (long long i = tid; i < TK; i += 1024) atomicAdd(&s_cnt[a.topk_idx[i]], 1);
    __syncthreads();
    if (tid == 0) {
        int acc = 0, cacc = 0;
        for (int e = 0; e < E; ++e) {
            a.counts[e] = s_cnt[e];
            a.offsets[e] = acc;
            a.chunk_start[e] = cacc;
            s_base[e] = acc;
            acc += s_cnt[e];
            cacc += (s_cnt[e] + a.chunk_rows - 1) / a.chunk_rows;
        }
        a.chunk_start[E] = cacc;
        for (int s = 0; s <= a.S; ++s) a.offsets[E + s] = acc + s * T;
    }
    // group order: longest first, lower index on ties
    for (int g = tid; g < E + a.S; g += 1024) {
        const int cg = g < E ? s_cnt[g] : T;
        int rank = 0;
        for (int h = 0; h < E + a.S; ++h) {
            const int ch = h < E ? s_cnt[h] : T;
            rank += (ch > cg) || (ch == cg && h < g);
        }
        a.gorder[rank] = g;
    }
    __syncthreads();
    for (int c0 = 0; c0 < T; c0 += 1024) {
        for (int q = tid; q < E * 32; q += 1024) (&s_mask[0][0])[q] = 0u;
        __syncthreads();
        const int t = c0 + tid;
        const int word = tid >> 5, bit = tid & 31;
        if (t < T)
            for (int j = 0; j < k; ++j) atomicOr(&s_mask[a.topk_idx[(size_t)t * k + j]][word], 1u << bit);
        __syncthreads();
        if (t < T) {
            for (int j = 0; j < k; ++j) {
                const int e = a.topk_idx[(size_t)t * k + j];
                int rank = __popc(s_mask[e][word] & ((1u << bit) - 1u));
                for (int w = 0; w < word; ++w) rank += __popc(s_mask[e][w]);
                const int pos = s_base[e] + rank;
                const int s = t * k + j;
                a.perm[pos] = s;
                a.inv_perm[s] = pos;
                a.row_token[pos] = t;
                a.row_slot[pos] = t * kk + j;
                a.row_w[pos] = a.topk_w[s];
            }
        }
        __syncthreads();
        for (int e = tid; e < E; e += 1024) {
            int n = 0;
            for (int w = 0; w < 32; ++w) n += __popc(s_mask[e][w]);
            s_base[e] += n;
        }
        __syncthreads();
    }
    // shared experts: every token, in token order, weight 1
    for (long long r = tid; r < (long long)a.S * T; r += 1024) {
        const int s = (int)(r / T), t = (int)(r % T);
        const long long pos = TK + r;
        a.row_token[pos] = t;
        a.row_slot[pos] = t * kk + k + s;
        a.row_w[pos] = 1.0f;
    }
}

}  // namespace mok
