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
// (so the same bits): eight warps per item for the split schedule's kernel
// below, one warp per item streaming through shared memory for the persistent
// kernel (drouter_stream, at the end of this file).

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

__device__ __forceinline__ void drouter_reduce_elem(long long i, const float *__restrict__ partial,
                                                   const int *__restrict__ chunk_start, float *__restrict__ dWr, int H)
{
    const int e = (int)(i / H), h = (int)(i % H);
    float s = 0.0f;
    for (int c = chunk_start[e]; c < chunk_start[e + 1]; ++c) s += partial[(size_t)c * H + h];
    dWr[i] = s;
}

// The same reduction in the persistent kernel: four columns per thread and four
// independent column groups in flight (one dependent load at a time per thread
// cannot hide the latency with 8 warps per SM); each element still sums its
// chunks in ascending order from 0 (same bits).
__device__ __forceinline__ void drouter_reduce_stream(const float *__restrict__ partial,
                                                      const int *__restrict__ chunk_start, float *__restrict__ dWr,
                                                      int H, int E)
{
    constexpr int U = 4;
    const long long nq = static_cast<long long>(E) * H / 4;
    const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
    for (long long q0 = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; q0 < nq; q0 += U * stride) {
        int c0[U], c1[U];
        long long i4[U];
        float4 acc[U];
        int nmax = 0;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long q = q0 + u * stride;
            i4[u] = q * 4;
            c0[u] = c1[u] = 0;
            if (q < nq) {
                const int e = static_cast<int>(i4[u] / H);
                c0[u] = chunk_start[e];
                c1[u] = chunk_start[e + 1];
            }
            acc[u] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            nmax = max(nmax, c1[u] - c0[u]);
        }
        for (int j = 0; j < nmax; ++j) {
            float4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c0[u] + j < c1[u])
                    v[u] = *reinterpret_cast<const float4 *>(partial + static_cast<size_t>(c0[u] + j) * H + i4[u] % H);
#pragma unroll
            for (int u = 0; u < U; ++u)
                if (c0[u] + j < c1[u]) {
                    acc[u].x += v[u].x; acc[u].y += v[u].y; acc[u].z += v[u].z; acc[u].w += v[u].w;
                }
        }
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (q0 + u * stride < nq) *reinterpret_cast<float4 *>(dWr + i4[u]) = acc[u];
    }
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


// ---- the same sums in the persistent kernels --------------------------------
// A persistent CTA has 8 warps per SM, far too few to hide HBM latency with the
// one-thread-per-element code above (the split kernels rely on 64 resident warps
// per SM).  Here every thread streams its own 16-byte pieces through a private
// ring of shared-memory slots with cp.async, NS units deep (up to 6), so the loads of the
// next NS-1 units are in flight while a unit is summed.  A thread reads back only
// the bytes it copied itself, so no barrier is needed between copy and use.  The
// arithmetic per output column is that of combine_elem / dx_combine_elem /
// drouter_partial_kernel, in the same order (same bits).
//   ring: `ring_bytes` of shared memory; slot (stage s, row j) of thread tid at
//   ring + ((s * R + j) * blockDim.x + tid) * 16 for R rows per unit.

__device__ __forceinline__ uint8_t *stream_slot(uint8_t *ring, int s, int R, int j)
{
    return ring + ((static_cast<size_t>(s) * R + j) * blockDim.x + threadIdx.x) * 16;
}

// stages that fit: units of R rows of 16 bytes per thread, at most 6
__device__ __forceinline__ int stream_stages(int R, int ring_bytes)
{
    const int ns = ring_bytes / (R * 16 * static_cast<int>(blockDim.x));
    return ns < 1 ? 1 : (ns > 6 ? 6 : ns);
}

template <int EPU>
__device__ __forceinline__ void slot_values(const uint8_t *p, float (&v)[EPU])
{
    if constexpr (EPU == 4) {
        const float4 a = *reinterpret_cast<const float4 *>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else {
        unpack8(*reinterpret_cast<const uint4 *>(p), v);
    }
}

template <int EPU>
__device__ __forceinline__ void store_bf16(__nv_bfloat16 *dst, const float (&v)[EPU])
{
    if constexpr (EPU == 4) {
        *reinterpret_cast<uint2 *>(dst) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
    } else {
        *reinterpret_cast<uint4 *>(dst) = pack8(v);
    }
}

// Forward combine: warp = token (warps take tokens in turn), lane = 16-byte column
// units lane, lane + 32, ...  The token's routing weights sit in lanes 0..k-1; the
// next token's are loaded while this one streams.
template <class Slot, int NS>
__device__ __forceinline__ void combine_stream_ns(const Slot *__restrict__ O, const float *__restrict__ topk_w,
                                                  __nv_bfloat16 *__restrict__ y, int T, int H, int k, int S,
                                                  uint8_t *ring)
{
    constexpr int EPU = 16 / sizeof(Slot);
    const int lane = threadIdx.x & 31;
    const int nw = gridDim.x * (blockDim.x >> 5);
    const int kk = k + S, units = H / (32 * EPU);
    int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    float wn = t < T && lane < k ? topk_w[static_cast<size_t>(t) * k + lane] : 0.0f;
    for (; t < T; t += nw) {
        const float wc = wn;
        if (t + nw < T && lane < k) wn = topk_w[static_cast<size_t>(t + nw) * k + lane];
        const Slot *rows = O + static_cast<size_t>(t) * kk * H + lane * EPU;
        auto issue = [&](int u) {
            for (int j = 0; j < kk; ++j)
                cp_async16(stream_slot(ring, u % NS, kk, j), rows + static_cast<size_t>(j) * H + u * 32 * EPU);
        };
#pragma unroll
        for (int u = 0; u < NS - 1; ++u) {
            if (u < units) issue(u);
            cp_async_commit();
        }
        for (int u = 0; u < units; ++u) {
            if (u + NS - 1 < units) issue(u + NS - 1);
            cp_async_commit();
            cp_async_wait<NS - 1>();
            float acc[EPU];
#pragma unroll
            for (int q = 0; q < EPU; ++q) acc[q] = 0.0f;
            for (int j = 0; j < kk; ++j) {
                const float w = __shfl_sync(0xffffffffu, wc, j < k ? j : 0);
                float v[EPU];
                slot_values<EPU>(stream_slot(ring, u % NS, kk, j), v);
#pragma unroll
                for (int q = 0; q < EPU; ++q) acc[q] = fmaf(j < k ? w : 1.0f, v[q], acc[q]);
            }
            store_bf16<EPU>(y + static_cast<size_t>(t) * H + u * 32 * EPU + lane * EPU, acc);
        }
    }
    cp_async_wait<0>();
}

template <class Slot>
__device__ __forceinline__ void combine_stream(const Slot *__restrict__ O, const float *__restrict__ topk_w,
                                               __nv_bfloat16 *__restrict__ y, int T, int H, int k, int S,
                                               uint8_t *ring, int ring_bytes)
{
    switch (stream_stages(k + S, ring_bytes)) {
    case 1: combine_stream_ns<Slot, 1>(O, topk_w, y, T, H, k, S, ring); break;
    case 2: combine_stream_ns<Slot, 2>(O, topk_w, y, T, H, k, S, ring); break;
    case 3: combine_stream_ns<Slot, 3>(O, topk_w, y, T, H, k, S, ring); break;
    case 4: combine_stream_ns<Slot, 4>(O, topk_w, y, T, H, k, S, ring); break;
    case 5: combine_stream_ns<Slot, 5>(O, topk_w, y, T, H, k, S, ring); break;
    default: combine_stream_ns<Slot, 6>(O, topk_w, y, T, H, k, S, ring); break;
    }
}

// dx sum: as combine_stream, with the token's k router-weight rows Wr[idx_j]
// streamed beside its k + S dX slot rows (R = 2k + S rows per unit).
template <int NS>
__device__ __forceinline__ void dx_stream_ns(const float *__restrict__ dXs, const float *__restrict__ dl,
                                             const int *__restrict__ topk_idx, const float *__restrict__ router_w,
                                             __nv_bfloat16 *__restrict__ dx, int T, int H, int k, int S,
                                             uint8_t *ring)
{
    const int lane = threadIdx.x & 31;
    const int nw = gridDim.x * (blockDim.x >> 5);
    const int kk = k + S, R = kk + k, units = H / 128;
    int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    float dn = 0.0f;
    int en = 0;
    if (t < T && lane < k) {
        dn = dl[static_cast<size_t>(t) * k + lane];
        en = topk_idx[static_cast<size_t>(t) * k + lane];
    }
    for (; t < T; t += nw) {
        const float dc = dn;
        const int ec = en;
        if (t + nw < T && lane < k) {
            dn = dl[static_cast<size_t>(t + nw) * k + lane];
            en = topk_idx[static_cast<size_t>(t + nw) * k + lane];
        }
        const float *rows = dXs + static_cast<size_t>(t) * kk * H + lane * 4;
        auto issue = [&](int u) {
            for (int j = 0; j < kk; ++j)
                cp_async16(stream_slot(ring, u % NS, R, j), rows + static_cast<size_t>(j) * H + u * 128);
            for (int j = 0; j < k; ++j) {
                const int e = __shfl_sync(0xffffffffu, ec, j);
                cp_async16(stream_slot(ring, u % NS, R, kk + j), router_w + static_cast<size_t>(e) * H + u * 128 +
                                                                     lane * 4);
            }
        };
#pragma unroll
        for (int u = 0; u < NS - 1; ++u) {
            if (u < units) issue(u);
            cp_async_commit();
        }
        for (int u = 0; u < units; ++u) {
            if (u + NS - 1 < units) issue(u + NS - 1);
            cp_async_commit();
            cp_async_wait<NS - 1>();
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int j = 0; j < kk; ++j) {
                float v[4];
                slot_values<4>(stream_slot(ring, u % NS, R, j), v);
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] += v[q];
            }
            for (int j = 0; j < k; ++j) {
                const float d = __shfl_sync(0xffffffffu, dc, j);
                float w[4];
                slot_values<4>(stream_slot(ring, u % NS, R, kk + j), w);
#pragma unroll
                for (int q = 0; q < 4; ++q) r[q] = fmaf(d, w[q], r[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] += r[q];
            store_bf16<4>(dx + static_cast<size_t>(t) * H + u * 128 + lane * 4, acc);
        }
    }
    cp_async_wait<0>();
}

// The same sum for k <= 8 (the DeepSeek-V3 layer): only the k + S dX rows (HBM)
// go through the ring, twice as deep; the token's k router-weight rows (L2-resident)
// come into registers with plain loads one unit ahead.
template <int NS>
__device__ __forceinline__ void dx_stream_k8_ns(const float *__restrict__ dXs, const float *__restrict__ dl,
                                                const int *__restrict__ topk_idx, const float *__restrict__ router_w,
                                                __nv_bfloat16 *__restrict__ dx, int T, int H, int k, int S,
                                                uint8_t *ring)
{
    constexpr int KM = 8;
    const int lane = threadIdx.x & 31;
    const int nw = gridDim.x * (blockDim.x >> 5);
    const int kk = k + S, units = H / 128;
    int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    float dn = 0.0f;
    int en = 0;
    if (t < T && lane < k) {
        dn = dl[static_cast<size_t>(t) * k + lane];
        en = topk_idx[static_cast<size_t>(t) * k + lane];
    }
    for (; t < T; t += nw) {
        const float dc = dn;
        const int ec = en;
        if (t + nw < T && lane < k) {
            dn = dl[static_cast<size_t>(t + nw) * k + lane];
            en = topk_idx[static_cast<size_t>(t + nw) * k + lane];
        }
        const float *rows = dXs + static_cast<size_t>(t) * kk * H + lane * 4;
        const float *wrow[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j)
            wrow[j] = router_w + static_cast<size_t>(__shfl_sync(0xffffffffu, ec, j < k ? j : 0)) * H + lane * 4;
        float4 wn[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) wn[j] = j < k ? __ldg(reinterpret_cast<const float4 *>(wrow[j])) : float4{};
        auto issue = [&](int u) {
            for (int j = 0; j < kk; ++j)
                cp_async16(stream_slot(ring, u % NS, kk, j), rows + static_cast<size_t>(j) * H + u * 128);
        };
#pragma unroll
        for (int u = 0; u < NS - 1; ++u) {
            if (u < units) issue(u);
            cp_async_commit();
        }
        for (int u = 0; u < units; ++u) {
            if (u + NS - 1 < units) issue(u + NS - 1);
            cp_async_commit();
            float4 wc[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) wc[j] = wn[j];
            if (u + 1 < units) {
#pragma unroll
                for (int j = 0; j < KM; ++j)
                    if (j < k) wn[j] = __ldg(reinterpret_cast<const float4 *>(wrow[j] + (u + 1) * 128));
            }
            cp_async_wait<NS - 1>();
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f}, r[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            for (int j = 0; j < kk; ++j) {
                float v[4];
                slot_values<4>(stream_slot(ring, u % NS, kk, j), v);
#pragma unroll
                for (int q = 0; q < 4; ++q) acc[q] += v[q];
            }
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < k) {
                    const float d = __shfl_sync(0xffffffffu, dc, j);
                    r[0] = fmaf(d, wc[j].x, r[0]);
                    r[1] = fmaf(d, wc[j].y, r[1]);
                    r[2] = fmaf(d, wc[j].z, r[2]);
                    r[3] = fmaf(d, wc[j].w, r[3]);
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] += r[q];
            store_bf16<4>(dx + static_cast<size_t>(t) * H + u * 128 + lane * 4, acc);
        }
    }
    cp_async_wait<0>();
}

__device__ __forceinline__ void dx_stream(const float *__restrict__ dXs, const float *__restrict__ dl,
                                          const int *__restrict__ topk_idx, const float *__restrict__ router_w,
                                          __nv_bfloat16 *__restrict__ dx, int T, int H, int k, int S, uint8_t *ring,
                                          int ring_bytes)
{
    if (k <= 8) {
        switch (stream_stages(k + S, ring_bytes)) {
        case 1: dx_stream_k8_ns<1>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        case 2: dx_stream_k8_ns<2>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        case 3: dx_stream_k8_ns<3>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        case 4: dx_stream_k8_ns<4>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        case 5: dx_stream_k8_ns<5>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        default: dx_stream_k8_ns<6>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); return;
        }
    }
    switch (stream_stages(2 * k + S, ring_bytes)) {
    case 1: dx_stream_ns<1>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    case 2: dx_stream_ns<2>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    case 3: dx_stream_ns<3>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    case 4: dx_stream_ns<4>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    case 5: dx_stream_ns<5>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    default: dx_stream_ns<6>(dXs, dl, topk_idx, router_w, dx, T, H, k, S, ring); break;
    }
}

// Router-gradient partial sums: warp = item (row chunk, 256 columns), lane = 8
// columns.  The item's rows run in units of 8 (one row per residue r0 + w mod 8),
// kDrouterStages units deep; a warp-private table in shared memory holds each row's token
// and dl, loaded once per item.  Sums per residue in ascending row order, then
// over the residues in order of w, as drouter_partial_kernel.
//   smem: the ring (kDrouterStages stages x 8 rows x 16 bytes per thread), then the warps'
//   row tables (kDrouterMaxRows x 8 bytes per warp), then chunk_start and offsets
//   ((E + 1) ints each).  Needs drouter_stream_bytes(E) bytes.
constexpr int kDrouterMaxRows = 256;             // rows per chunk at most
constexpr int kDrouterStages = 6;
__host__ __device__ constexpr int drouter_stream_bytes(int threads, int E)
{
    return kDrouterStages * 8 * 16 * threads + threads / 32 * kDrouterMaxRows * 8 + 2 * (E + 1) * 4;
}

__device__ __forceinline__ void drouter_stream(const __nv_bfloat16 *__restrict__ x, const float *__restrict__ dl,
                                               const int *__restrict__ offsets, const int *__restrict__ chunk_start,
                                               const int *__restrict__ perm, float *__restrict__ partial, int H, int E,
                                               int k, int chunk_rows, uint8_t *smem)
{
    constexpr int NS = kDrouterStages;
    const int nthr = blockDim.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint8_t *ring = smem;
    int *tab_tok = reinterpret_cast<int *>(smem + NS * 8 * 16 * nthr) + warp * 2 * kDrouterMaxRows;
    float *tab_d = reinterpret_cast<float *>(tab_tok + kDrouterMaxRows);
    int *s_cs = reinterpret_cast<int *>(smem + NS * 8 * 16 * nthr) + (nthr >> 5) * 2 * kDrouterMaxRows;
    int *s_off = s_cs + E + 1;
    for (int i = threadIdx.x; i <= E; i += nthr) {
        s_cs[i] = chunk_start[i];
        s_off[i] = offsets[i];
    }
    __syncthreads();
    const int hb = H / 256;
    const int n_items = s_cs[E] * hb;
    const int nw = gridDim.x * (nthr >> 5);
    for (int item = blockIdx.x * (nthr >> 5) + warp; item < n_items; item += nw) {
        const int chunk = item / hb, h0 = (item - chunk * hb) * 256;
        int r1;
        const int r0 = drouter_chunk_rows(chunk, s_off, s_cs, E, chunk_rows, r1);
        const int nrows = r1 - r0, units = (nrows + 7) >> 3;
        int sv[kDrouterMaxRows / 32];
        float dv[kDrouterMaxRows / 32];
#pragma unroll
        for (int m = 0; m < kDrouterMaxRows / 32; ++m)
            sv[m] = lane + 32 * m < nrows ? perm[r0 + lane + 32 * m] : 0;
#pragma unroll
        for (int m = 0; m < kDrouterMaxRows / 32; ++m) dv[m] = lane + 32 * m < nrows ? dl[sv[m]] : 0.0f;
        __syncwarp();                              // the previous item's table reads are done
#pragma unroll
        for (int m = 0; m < kDrouterMaxRows / 32; ++m)
            if (lane + 32 * m < nrows) {
                tab_tok[lane + 32 * m] = sv[m] / k;
                tab_d[lane + 32 * m] = dv[m];
            }
        __syncwarp();
        const __nv_bfloat16 *xc = x + h0 + lane * 8;
        auto issue = [&](int u) {
            for (int w = 0; w < 8; ++w) {
                const int i = u * 8 + w;
                if (i < nrows) cp_async16(stream_slot(ring, u % NS, 8, w), xc + static_cast<size_t>(tab_tok[i]) * H);
            }
        };
        float acc[8][8];
#pragma unroll
        for (int w = 0; w < 8; ++w)
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[w][q] = 0.0f;
#pragma unroll
        for (int u = 0; u < NS - 1; ++u) {
            if (u < units) issue(u);
            cp_async_commit();
        }
        for (int u = 0; u < units; ++u) {
            if (u + NS - 1 < units) issue(u + NS - 1);
            cp_async_commit();
            cp_async_wait<NS - 1>();
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                const int i = u * 8 + w;
                if (i < nrows) {
                    const float d = tab_d[i];
                    float v[8];
                    slot_values<8>(stream_slot(ring, u % NS, 8, w), v);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc[w][q] = fmaf(d, v[q], acc[w][q]);
                }
            }
        }
        float sum[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float s = 0.0f;
#pragma unroll
            for (int w = 0; w < 8; ++w) s += acc[w][q];
            sum[q] = s;
        }
        float *dst = partial + static_cast<size_t>(chunk) * H + h0 + lane * 8;
        reinterpret_cast<float4 *>(dst)[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
        reinterpret_cast<float4 *>(dst)[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
    }
    cp_async_wait<0>();
}

}  // namespace mok
