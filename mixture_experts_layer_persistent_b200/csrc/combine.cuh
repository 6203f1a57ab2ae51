// combine.cuh -- the HBM-bound steps: the fixed-order weighted k-sum of the
// forward, the per-slot routing gradient, the router weight gradient and the
// final dx sum of the backward.  All sums run in a fixed order with no
// floating-point atomics, so results are bit-reproducible.
#pragma once
#include "ptx.cuh"

namespace mok {

__device__ __forceinline__ void unpack8(const uint4 u, float (&v)[8])
{
    v[0] = bf16_lo(u.x); v[1] = bf16_hi(u.x); v[2] = bf16_lo(u.y); v[3] = bf16_hi(u.y);
    v[4] = bf16_lo(u.z); v[5] = bf16_hi(u.z); v[6] = bf16_lo(u.w); v[7] = bf16_hi(u.w);
}

__device__ __forceinline__ void load8(const float *p, float (&v)[8])
{
    const float4 a = reinterpret_cast<const float4 *>(p)[0], b = reinterpret_cast<const float4 *>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16 *p, float (&v)[8])
{
    unpack8(*reinterpret_cast<const uint4 *>(p), v);
}

__device__ __forceinline__ uint4 pack8(const float (&v)[8])
{
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    return u;
}

// y[t] = sum_{j<k} w[t,j] O[t,j] (ascending j) + sum_s O[t,k+s] (ascending s), fp32, -> bf16.
// Thread = 8 columns of one token (16-byte loads).
// O: fp32 slot rows (BF16 layer) or bf16 slot rows (MXFP8 forward)
// B slot rows' loads are issued before their sums, which still run in ascending j
// (B = 4 in the split kernel, where occupancy keeps many threads in flight; 8 in
// the persistent kernel, whose 320 threads per SM need more loads each)
template <class Slot, int B = 4>
__device__ __forceinline__ void combine_elem(long long i, const Slot *__restrict__ O,
                                             const float *__restrict__ topk_w, __nv_bfloat16 *__restrict__ y,
                                             int H, int k, int S)
{
    const int cpr = H / 8;
    const int t = (int)(i / cpr), c = (int)(i % cpr) * 8;
    const int kk = k + S;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const Slot *row = O + (size_t)t * kk * H + c;
    int j = 0;
    for (; j + B <= kk; j += B) {
        float v[B][8], w[B];
#pragma unroll
        for (int u = 0; u < B; ++u) {
            w[u] = j + u < k ? topk_w[(size_t)t * k + j + u] : 1.0f;
            load8(row + (size_t)(j + u) * H, v[u]);
        }
#pragma unroll
        for (int u = 0; u < B; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(w[u], v[u][q], acc[q]);
    }
    for (; j < kk; ++j) {
        const float w = j < k ? topk_w[(size_t)t * k + j] : 1.0f;
        float v[8];
        load8(row + (size_t)j * H, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(w, v[q], acc[q]);
    }
    *reinterpret_cast<uint4 *>(y + (size_t)t * H + c) = pack8(acc);
}

template <class Slot>
__global__ void __launch_bounds__(256) combine_kernel(const Slot *__restrict__ O,
                                                      const float *__restrict__ topk_w,
                                                      __nv_bfloat16 *__restrict__ y, int T, int H, int k, int S)
{
    griddep_enter();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (long long)T * (H / 8)) combine_elem(i, O, topk_w, y, H, k, S);
}

// Backward, per token: G_j = <dy[t], o_j> (j < k), summed in a fixed order from the
// per-N-tile partials <dy W_down, h> that the down dgrad GEMM's epilogue wrote for
// the slot's sorted row (o_j = h_j W_down^T, so the two are equal), then the logit
// gradient
//   softmax: dl_j = w_j (G_j - sum_i q_i G_i),             q = w / routed_scale
//   sigmoid: dl_j = rho/S (G_j - sum_i q_i G_i) s_j (1 - s_j), S = sum of selected s
// One thread per token.
__device__ __forceinline__ void slot_grad_token(int t, const float *__restrict__ gpart, int n_parts,
                                                const int *__restrict__ inv_perm, const float *__restrict__ topk_w,
                                                const float *__restrict__ topk_p, float *__restrict__ dl, int k,
                                                int score_fn, float routed_scale)
{
    float G[16], q[16];
    float gbar = 0.0f, S_ = 0.0f;
    for (int j = 0; j < k; ++j) {
        const float *gp = gpart + (size_t)inv_perm[(size_t)t * k + j] * n_parts;
        float v = 0.0f;
        for (int p = 0; p < n_parts; ++p) v += gp[p];
        G[j] = v;
        q[j] = topk_w[(size_t)t * k + j] / routed_scale;
        gbar = fmaf(q[j], G[j], gbar);
        S_ += topk_p[(size_t)t * k + j];
    }
    for (int j = 0; j < k; ++j) {
        float r;
        if (score_fn == 0) {
            r = topk_w[(size_t)t * k + j] * (G[j] - gbar);
        } else {
            const float s = topk_p[(size_t)t * k + j];
            r = routed_scale / S_ * (G[j] - gbar) * s * (1.0f - s);
        }
        dl[(size_t)t * k + j] = r;
    }
}

__global__ void __launch_bounds__(256) slot_grad_kernel(const float *__restrict__ gpart, int n_parts,
                                                        const int *__restrict__ inv_perm,
                                                        const float *__restrict__ topk_w,
                                                        const float *__restrict__ topk_p, float *__restrict__ dl,
                                                        int T, int k, int score_fn, float routed_scale)
{
    griddep_enter();
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t < T) slot_grad_token(t, gpart, n_parts, inv_perm, topk_w, topk_p, dl, k, score_fn, routed_scale);
}

// Router weight gradient, pass 1: for each chunk of up to `chunk_rows` sorted
// rows of one expert and 256 columns, partial[chunk, cols] = sum over the
// chunk's rows of dl(row) x[token(row), cols], in a fixed order: the rows
// r0 + w, r0 + w + 8, ... (w = 0..7) are summed separately in ascending order,
// then the eight sums in order of w.  Two implementations with that same order
// (so the same bits): eight warps per item for the split schedule's kernel, a
// team of two warps per item for the persistent kernel.

__device__ __forceinline__ int drouter_chunk_rows(int chunk, const int *__restrict__ offsets,
                                                  const int *__restrict__ chunk_start, int E, int chunk_rows, int &r1)
{
    int lo = 0, hi = E - 1;     // expert owning this chunk: largest e with chunk_start[e] <= chunk
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (chunk_start[mid] <= chunk) lo = mid; else hi = mid - 1;
    }
    const int r0 = offsets[lo] + (chunk - chunk_start[lo]) * chunk_rows;
    r1 = min(offsets[lo + 1], r0 + chunk_rows);
    return r0;
}

// split schedule: one item per block of 256 threads, warp w sums the rows of residue w
__global__ void __launch_bounds__(256) drouter_partial_kernel(const __nv_bfloat16 *__restrict__ x,
                                                              const float *__restrict__ dl,
                                                              const int *__restrict__ offsets,
                                                              const int *__restrict__ chunk_start,
                                                              const int *__restrict__ perm,
                                                              float *__restrict__ partial, int H, int E, int k,
                                                              int chunk_rows)
{
    griddep_enter();
    __shared__ float s_acc[8][256];
    const int chunk = blockIdx.x;
    const int h0 = blockIdx.y * 256;
    if (chunk >= chunk_start[E]) return;
    int r1;
    const int r0 = drouter_chunk_rows(chunk, offsets, chunk_start, E, chunk_rows, r1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int r = r0 + warp; r < r1; r += 8) {
        const int s = perm[r];                  // t * k + slot
        const float d = dl[s];
        float v[8];
        unpack8(*reinterpret_cast<const uint4 *>(x + (size_t)(s / k) * H + h0 + lane * 8), v);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(d, v[q], acc[q]);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) s_acc[warp][lane * 8 + q] = acc[q];
    __syncthreads();
    float s = 0.0f;
    for (int w = 0; w < 8; ++w) s += s_acc[w][threadIdx.x];
    partial[(size_t)chunk * H + h0 + threadIdx.x] = s;
}

// persistent schedule: a team of two warps per item (warp half h sums residues
// 4h .. 4h+3, four rows in flight); s_acc: the team's [8][256] floats of shared
// memory; bar: the team's named barrier (64 threads)
__device__ __forceinline__ void drouter_partial_team(int chunk, int h0, int half, int lane, int bar,
                                                     const __nv_bfloat16 *__restrict__ x, const float *__restrict__ dl,
                                                     const int *__restrict__ offsets,
                                                     const int *__restrict__ chunk_start,
                                                     const int *__restrict__ perm, float *__restrict__ partial,
                                                     int H, int E, int k, int chunk_rows, float (*s_acc)[256])
{
    int r1;
    const int r0 = drouter_chunk_rows(chunk, offsets, chunk_start, E, chunk_rows, r1);
    float acc[4][8];
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[w][q] = 0.0f;
    for (int r = r0 + 4 * half; r < r1; r += 8) {
        float v[4][8], d[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            if (r + w < r1) {
                const int s = perm[r + w];
                d[w] = dl[s];
                unpack8(*reinterpret_cast<const uint4 *>(x + (size_t)(s / k) * H + h0 + lane * 8), v[w]);
            }
        }
#pragma unroll
        for (int w = 0; w < 4; ++w)
            if (r + w < r1)
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[w][q] = fmaf(d[w], v[w][q], acc[w][q]);
    }
#pragma unroll
    for (int w = 0; w < 4; ++w)
#pragma unroll
        for (int q = 0; q < 8; ++q) s_acc[4 * half + w][lane * 8 + q] = acc[w][q];
    asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
    for (int c = half * 32 + lane; c < 256; c += 64) {
        float s = 0.0f;
        for (int w = 0; w < 8; ++w) s += s_acc[w][c];
        partial[(size_t)chunk * H + h0 + c] = s;
    }
    asm volatile("bar.sync %0, 64;" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void drouter_reduce_elem(long long i, const float *__restrict__ partial,
                                                   const int *__restrict__ chunk_start, float *__restrict__ dWr, int H)
{
    const int e = (int)(i / H), h = (int)(i % H);
    float s = 0.0f;
    for (int c = chunk_start[e]; c < chunk_start[e + 1]; ++c) s += partial[(size_t)c * H + h];
    dWr[i] = s;
}

__global__ void __launch_bounds__(256) drouter_reduce_kernel(const float *__restrict__ partial,
                                                             const int *__restrict__ chunk_start,
                                                             float *__restrict__ dWr, int H, int E)
{
    griddep_enter();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (long long)E * H) drouter_reduce_elem(i, partial, chunk_start, dWr, H);
}

// dx[t] = sum_j dXs[t, j] (ascending j over routed then shared slots)
//         + sum_{j<k} dl[t, j] router_w[idx[t, j]]   -> bf16.
template <int B = 4>
__device__ __forceinline__ void dx_combine_elem(long long i, const float *__restrict__ dXs,
                                                const float *__restrict__ dl, const int *__restrict__ topk_idx,
                                                const float *__restrict__ router_w, __nv_bfloat16 *__restrict__ dx,
                                                int H, int k, int S)
{
    const int cpr = H / 8;
    const int t = (int)(i / cpr), c = (int)(i % cpr) * 8;
    const int kk = k + S;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const float *row = dXs + (size_t)t * kk * H + c;
    int j = 0;
    for (; j + B <= kk; j += B) {                  // B rows' loads in flight, sums in ascending j
        float v[B][8];
#pragma unroll
        for (int u = 0; u < B; ++u) load8(row + (size_t)(j + u) * H, v[u]);
#pragma unroll
        for (int u = 0; u < B; ++u)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] += v[u][q];
    }
    for (; j < kk; ++j) {
        float v[8];
        load8(row + (size_t)j * H, v);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] += v[q];
    }
    float r[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
        const float d = dl[(size_t)t * k + j];
        const float *wr = router_w + (size_t)topk_idx[(size_t)t * k + j] * H + c;
        const float4 w0 = *reinterpret_cast<const float4 *>(wr);
        const float4 w1 = *reinterpret_cast<const float4 *>(wr + 4);
        r[0] = fmaf(d, w0.x, r[0]); r[1] = fmaf(d, w0.y, r[1]); r[2] = fmaf(d, w0.z, r[2]); r[3] = fmaf(d, w0.w, r[3]);
        r[4] = fmaf(d, w1.x, r[4]); r[5] = fmaf(d, w1.y, r[5]); r[6] = fmaf(d, w1.z, r[6]); r[7] = fmaf(d, w1.w, r[7]);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] += r[q];
    *reinterpret_cast<uint4 *>(dx + (size_t)t * H + c) = pack8(acc);
}

__global__ void __launch_bounds__(256) dx_combine_kernel(const float *__restrict__ dXs,
                                                         const float *__restrict__ dl,
                                                         const int *__restrict__ topk_idx,
                                                         const float *__restrict__ router_w,
                                                         __nv_bfloat16 *__restrict__ dx, int T, int H, int k, int S)
{
    griddep_enter();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < (long long)T * (H / 8)) dx_combine_elem(i, dXs, dl, topk_idx, router_w, dx, H, k, S);
}

}  // namespace mok
