// route.cuh -- router logits, scoring and top-k selection, and the
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

struct RouteArgs {
    const __nv_bfloat16 *x;     // [T, H]
    const float *router_w;      // [E, H]
    const float *e_bias;        // [E] or null
    const float *logit_bias;    // [E] or null
    int T, H, E, k;
    int score_fn, n_group, topk_group;
    float routed_scale;
    int *topk_idx;              // [T, k]
    float *topk_w;              // [T, k]
    float *topk_p;              // [T, k] sigmoid score s (sigmoid) or w / routed_scale (softmax)
};

constexpr int kRouteTokens = 32;   // tokens per block
constexpr int kRouteHC = 32;       // H chunk staged in shared memory
constexpr int kRoutePad = 36;      // padded row stride (floats)

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

// Block: 256 threads, 32 tokens.  Thread (eg = tid % 64, tg = tid / 64) owns
// experts eg + 64 i (i < 4) and tokens 8 tg .. 8 tg + 7: 32 fp32 dot products
// over H, each accumulated in ascending h.
__global__ void __launch_bounds__(256) router_kernel(const RouteArgs a)
{
    __shared__ __align__(16) float s_w[256 * kRoutePad];              // router rows chunk, later logits
    __shared__ __align__(16) float s_x[kRouteTokens * kRoutePad];
    const int tid = threadIdx.x;
    const int t0 = blockIdx.x * kRouteTokens;
    const int eg = tid & 63, tg = tid >> 6;
    const int E = a.E, H = a.H;
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;

    for (int h0 = 0; h0 < H; h0 += kRouteHC) {
        // stage router rows [E, 32] and x rows [32, 32] (as fp32)
        for (int q = tid; q < E * (kRouteHC / 4); q += 256) {
            const int e = q / (kRouteHC / 4), c4 = q % (kRouteHC / 4);
            const float4 v = *reinterpret_cast<const float4 *>(a.router_w + (size_t)e * H + h0 + c4 * 4);
            *reinterpret_cast<float4 *>(&s_w[e * kRoutePad + c4 * 4]) = v;
        }
        for (int q = tid; q < kRouteTokens * (kRouteHC / 8); q += 256) {
            const int tt = q / (kRouteHC / 8), c8 = q % (kRouteHC / 8);
            const int t = t0 + tt;
            float v[8];
            if (t < a.T) {
                const uint4 u = *reinterpret_cast<const uint4 *>(a.x + (size_t)t * H + h0 + c8 * 8);
                v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
                v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) s_x[tt * kRoutePad + c8 * 8 + i] = v[i];
        }
        __syncthreads();
#pragma unroll
        for (int hh = 0; hh < kRouteHC; hh += 4) {
            float4 xv[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) xv[j] = *reinterpret_cast<const float4 *>(&s_x[(tg * 8 + j) * kRoutePad + hh]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int e = eg + 64 * i;
                if (e < E) {
                    const float4 wv = *reinterpret_cast<const float4 *>(&s_w[e * kRoutePad + hh]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        float s = acc[i][j];
                        s = fmaf(xv[j].x, wv.x, s);
                        s = fmaf(xv[j].y, wv.y, s);
                        s = fmaf(xv[j].z, wv.z, s);
                        s = fmaf(xv[j].w, wv.w, s);
                        acc[i][j] = s;
                    }
                }
            }
        }
        __syncthreads();
    }
    // logits to shared memory: s_w[tt * 257 + e]
    float *s_lg = s_w;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int e = eg + 64 * i;
        if (e < E) {
            const float lb = a.logit_bias ? a.logit_bias[e] : 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) s_lg[(tg * 8 + j) * 257 + e] = acc[i][j] + lb;
        }
    }
    __syncthreads();

    // selection: warp w handles tokens w, w + 8, w + 16, w + 24
    const int warp = tid >> 5, lane = tid & 31;
    const int npl = (E + 31) / 32;
    for (int tt = warp; tt < kRouteTokens; tt += 8) {
        const int t = t0 + tt;
        if (t >= a.T) break;
        float *lg = s_lg + tt * 257;
        float sel[8], sc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = lane + 32 * i;
            sel[i] = -INFINITY;
            sc[i] = 0.0f;
            if (i < npl && e < E) {
                if (a.score_fn == 0) {
                    sel[i] = lg[e];
                } else {
                    const float s = 1.0f / (1.0f + expf(-lg[e]));
                    sc[i] = s;
                    sel[i] = s + (a.e_bias ? a.e_bias[e] : 0.0f);
                }
            }
        }
        if (a.n_group > 1 && a.topk_group < a.n_group) {
            // group score: sum of the two best selection scores of the group
            const int gs = E / a.n_group;
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = lane + 32 * i;
                if (i < npl && e < E) lg[e] = sel[i];   // reuse the logit row for selection scores
            }
            __syncwarp();
            float gsc = -INFINITY;
            if (lane < a.n_group) {
                float b1 = -INFINITY, b2 = -INFINITY;
                for (int m = 0; m < gs; ++m) {
                    const float v = lg[lane * gs + m];
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
            // owner retires the winner
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (lane + 32 * i == bi) sel[i] = -INFINITY;
            // the winner's weight ingredient: logit (softmax) or sigmoid score
            float wv = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (lane + 32 * i == bi) wv = a.score_fn == 0 ? s_lg[tt * 257 + bi] : sc[i];
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
