// ep.cuh -- expert parallelism: the rank-crossing steps of the forward.
//
// "Cursor åpner megakernelen…" (the pull-versus-push paragraph) and
// "Megakernels are dead and back…" ("Números de MoK"): the GPU that owns an
// expert pulls the token rows routed to it from the GPU that holds them, and
// pushes each expert output row back to that GPU, where the fixed-order k-sum
// runs.  Here rank r owns the routed experts [r E_loc, (r+1) E_loc) and every
// rank routes its own T tokens over all E experts (route.cuh, unchanged).
//
// The owner's sorted rows: for each of its experts j (ascending), the rows of
// every source rank s (ascending), each source's rows in its own dispatch
// order (token ascending), then the shared experts' rows of the owner's own
// tokens.  Every output row depends only on its own input row and the expert's
// weights, so the order changes no value: each rank's y equals the one-GPU
// layer's on its tokens, byte for byte.
//
// Peer buffers are addressed through plain pointers valid on this device (the
// owner's own buffers, another allocation on the same device, or another GPU's
// memory mapped into this process); loads and stores are ordinary global ones
// (no TMA, no multicast).  The calls of one phase must be complete on every
// rank before any rank starts the next phase; the caller orders them.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "mok.h"
#include "quant.cuh"

namespace mok {

constexpr int kEpMaxRanks = MOK_EP_MAX_RANKS;
// Row codes that cross ranks: (rank << kEpRankShift) | row on that rank
constexpr int kEpRankShift = 24;
constexpr int kEpRowMask = (1 << kEpRankShift) - 1;
constexpr int kEpMaxGroups = 256 + 4;   // routed experts of one rank + shared experts

// Every rank's routing record and slot rows, as this device addresses them.
struct EpView {
    const int *counts[kEpMaxRanks];     // [E] tokens of rank s per expert
    const int *offsets[kEpMaxRanks];    // [E + S + 1] rank s's sorted-row ranges
    const int *perm[kEpMaxRanks];       // [T k] rank s's sorted row -> t k + slot
    const float *topk_w[kEpMaxRanks];   // [T k] rank s's routing weights
    const int *topk_idx[kEpMaxRanks];   // [T k] rank s's selected experts
    float *O[kEpMaxRanks];              // [T, k + S, H] rank s's fp32 slot rows
};

struct EpArgs {
    int world, rank;
    int T, H, k, kk, S, E_loc;
    int rr_cap;            // routed rows this rank can receive: world T min(k, E_loc)
    int *seg;              // [E_loc world + 1] first sorted row of each (expert, source) segment; seg[n] = routed rows
    int *offsets;          // [E_loc + S + 1] the owner's group ranges (routed experts, then shared)
    int *row_token;        // [rows] row of x_recv each sorted row reads
    int *recv_idx;         // [world T] received row of (source rank, token), -1 if none
    int *uniq_src;         // [world T] (source rank << 24) | token of each received row
    int *n_recv;           // received rows (distinct (source rank, token) pairs)
    int *row_slot;         // [rows] (source rank << 24) | slot row t (k + S) + slot in that rank's O
    int *row_gdst;         // [routed rows] (source rank << 24) | the row's position in the source's sorted rows
    float *row_w;          // [rows] routing weight (1 for shared rows)
    int *gorder;           // [E_loc + S] the owner's groups by rows descending, index ascending
    float **push;          // [kEpMaxRanks] slot rows of every rank, for the push epilogue
    int *status;
};

// One block of 256 threads: segment sizes from every source's counts, their
// exclusive scan (ascending (expert, source)), the owner's group ranges and
// the push table.  E_loc * world = E <= 256 segments, one per thread.
// s_scan: 256 + 2 + kEpMaxGroups ints of shared memory.
__device__ __forceinline__ void ep_layout_block(const EpView &v, const EpArgs &a, int *s_scan)
{
    int &s_total = s_scan[256];
    int &s_bad = s_scan[257];
    int *s_rows = s_scan + 258;
    const int n = a.E_loc * a.world;
    const int i = threadIdx.x;
    int c = 0;
    if (i < n) {
        const int j = i / a.world, s = i - j * a.world;
        c = v.counts[s][a.rank * a.E_loc + j];
        if (c < 0 || c > a.T) c = -1;       // impossible count: reject the whole layout below
    }
    s_scan[i] = c;
    __syncthreads();
    // inclusive Hillis-Steele scan
    for (int d = 1; d < 256; d <<= 1) {
        const int add = i >= d ? s_scan[i - d] : 0;
        __syncthreads();
        s_scan[i] += add;
        __syncthreads();
    }
    if (i == 0) s_total = s_scan[n - 1];
    if (i == 0) s_bad = 0;
    __syncthreads();
    if (c < 0) atomicOr(&s_bad, 1);
    __syncthreads();
    // Bound every index the later steps use: a layout larger than the receive
    // buffers (impossible for counts written by the dispatch) becomes empty.
    const bool ok = !s_bad && s_total <= a.rr_cap;
    if (!ok && i == 0) atomicOr(a.status, MOK_STATUS_BAD_INDEX);
    const int total = ok ? s_total : 0;
    const int excl = ok ? s_scan[i] - c : 0;
    if (i < n) a.seg[i] = excl;
    if (i == 0) a.seg[n] = total;
    if (i < n && i % a.world == 0) a.offsets[i / a.world] = excl;
    if (i <= a.S) a.offsets[a.E_loc + i] = total + i * a.T;
    if (i < a.world) a.push[i] = v.O[i];
    // longest-first group order of the weight gradients (ties: lower index first)
    const int G = a.E_loc + a.S;
    for (int g = i; g < G; g += blockDim.x) {
        int rows = a.T;                                      // a shared group: the owner's T tokens
        if (g < a.E_loc) rows = ok ? s_scan[(g + 1) * a.world - 1] - (g ? s_scan[g * a.world - 1] : 0) : 0;
        s_rows[g] = rows;
    }
    __syncthreads();
    for (int g = i; g < G; g += blockDim.x) {
        int rank = 0;
        for (int h = 0; h < G; ++h) rank += s_rows[h] > s_rows[g] || (s_rows[h] == s_rows[g] && h < g);
        a.gorder[rank] = g;
    }
}

__global__ void __launch_bounds__(256) ep_layout_kernel(EpView v, EpArgs a)
{
    __shared__ int s_scan[256 + 2 + kEpMaxGroups];
    ep_layout_block(v, a, s_scan);
}

// The token rows the owner receives: every (source rank, token) pair with at
// least one selected expert on the owner, once, in (rank, token) order -- a token
// with several of its experts on one owner crosses the link once.  One block,
// each thread a run of consecutive pairs: count, block scan, write.
// Any block size that is a multiple of 32, up to 1024; s_warp: 32 ints of shared memory.
__device__ __forceinline__ void ep_unique_block(const EpView &v, const EpArgs &a, int *s_warp)
{
    const int nt = blockDim.x, nw = nt >> 5;
    const int n = a.world * a.T;
    const int per = (n + nt - 1) / nt;
    const int i0 = threadIdx.x * per, i1 = min(n, i0 + per);
    const int e0 = a.rank * a.E_loc, e1 = e0 + a.E_loc;
    auto wanted = [&](int i) {
        const int s = i / a.T, t = i - s * a.T;
        const int *idx = v.topk_idx[s] + (size_t)t * a.k;
        bool w = false;
#pragma unroll
        for (int j = 0; j < 16; ++j)             // k <= 16: every load issued before the compares
            if (j < a.k) {
                const int e = idx[j];
                w |= e >= e0 && e < e1;
            }
        return w;
    };
    // first pass: flags of this thread's run (kept in a mask while the run is at most 32 long)
    unsigned mask = 0;
    int cnt = 0;
    for (int i = i0; i < i1; ++i) {
        const bool w = wanted(i);
        if (w && i - i0 < 32) mask |= 1u << (i - i0);
        cnt += w;
    }
    // block-wide exclusive scan of the counts: within warps, then over the 32 warp sums
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int inc = cnt;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, inc, d);
        if (lane >= d) inc += o;
    }
    if (lane == 31) s_warp[wid] = inc;
    __syncthreads();
    if (wid == 0) {
        int ws = lane < nw ? s_warp[lane] : 0;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, ws, d);
            if (lane >= d) ws += o;
        }
        if (lane < nw) s_warp[lane] = ws;            // inclusive over warps
    }
    __syncthreads();
    int u = (wid ? s_warp[wid - 1] : 0) + inc - cnt;
    for (int i = i0; i < i1; ++i) {
        const bool w = i - i0 < 32 ? (mask >> (i - i0)) & 1u : wanted(i);
        if (w) {
            const int s = i / a.T;
            a.recv_idx[i] = u;
            a.uniq_src[u] = (s << kEpRankShift) | (i - s * a.T);
            ++u;
        } else {
            a.recv_idx[i] = -1;
        }
    }
    if (threadIdx.x == nt - 1) *a.n_recv = s_warp[nw - 1];
}

__global__ void __launch_bounds__(1024) ep_unique_kernel(EpView v, EpArgs a)
{
    __shared__ int s_warp[32];
    ep_unique_block(v, a, s_warp);
}

// Sorted rows of the owner.  Blocks [0, n): segment b = (expert j, source s)
// copies source s's rows of expert e = rank E_loc + j; blocks after those:
// the shared experts' rows of the owner's own tokens, 256 tokens per block.
__device__ __forceinline__ void ep_rows_block(const EpView &v, const EpArgs &a, int b)
{
    const int n = a.E_loc * a.world;
    if (b < n) {
        const int j = b / a.world, s = b - j * a.world;
        const int e = a.rank * a.E_loc + j;
        const int base = a.seg[b];
        const int cnt = a.seg[b + 1] - base;
        const int src0 = v.offsets[s][e];
        const int tk = a.T * a.k;
        // a range outside the source's rows (impossible for a record the dispatch wrote)
        // leaves every row of the segment in bounds: token 0, slot 0, weight 0
        const bool range_ok = src0 >= 0 && src0 + cnt <= tk;
        if (!range_ok && threadIdx.x == 0 && cnt > 0) atomicOr(a.status, MOK_STATUS_BAD_INDEX);
        for (int i = threadIdx.x; i < cnt; i += blockDim.x) {
            int q = range_ok ? v.perm[s][src0 + i] : 0;  // t k + slot on rank s
            if (q < 0 || q >= tk) {
                atomicOr(a.status, MOK_STATUS_BAD_INDEX);
                q = 0;
            }
            const int t = q / a.k, slot = q - t * a.k;
            const int r = base + i;
            int u = a.recv_idx[s * a.T + t];
            if (u < 0) {                                 // a row the selection does not list
                atomicOr(a.status, MOK_STATUS_BAD_INDEX);
                u = 0;
            }
            a.row_token[r] = a.T + u;
            a.row_slot[r] = (s << kEpRankShift) | (t * a.kk + slot);
            a.row_gdst[r] = (s << kEpRankShift) | (range_ok ? src0 + i : 0);
            a.row_w[r] = range_ok ? v.topk_w[s][q] : 0.0f;
        }
    } else {
        const int nb = (a.T + 255) / 256;
        const int sb = b - n;
        const int s2 = sb / nb;
        const int t = (sb - s2 * nb) * 256 + threadIdx.x;
        if (s2 < a.S && t < a.T) {
            const int r = a.seg[n] + s2 * a.T + t;
            a.row_token[r] = t;
            a.row_slot[r] = (a.rank << kEpRankShift) | (t * a.kk + a.k + s2);
            a.row_w[r] = 1.0f;
        }
    }
}

// blocks: E_loc world segments, then S ceil(T / 256) blocks of shared rows
__device__ __forceinline__ int ep_row_blocks(const EpArgs &a) { return a.E_loc * a.world + a.S * ((a.T + 255) / 256); }

__global__ void __launch_bounds__(256) ep_rows_kernel(EpView v, EpArgs a) { ep_rows_block(v, a, blockIdx.x); }

// Pull at dispatch: dst row t = the owner's own row t for t < T, dst row T + u =
// the u-th received (source rank, token) row (x, dy, or x's MXFP8 codes or scales).
// One warp per row, V-sized loads (16 or 8 bytes), four in flight per lane;
// every remote row crosses the link once.
struct EpPull {
    const uint8_t *src[kEpMaxRanks];   // every rank's token rows, row_bytes each
    uint8_t *dst;                      // [T + received rows, row_bytes]
    long long row_bytes;               // a multiple of sizeof(V)
    int T, world, rank;
    const int *n_recv;                 // received rows
    const int *row_src;                // (source rank << 24) | token of each received row
    int *status;
};

template <typename V>
__device__ __forceinline__ void ep_pull_rows(const EpPull &a, int warp, int n_warps, int lane)
{
    const int rows = a.T + min(*a.n_recv, a.world * a.T);
    const int vec = static_cast<int>(a.row_bytes / static_cast<long long>(sizeof(V)));
    for (int r = warp; r < rows; r += n_warps) {
        const uint8_t *src;
        if (r < a.T) {
            src = a.src[a.rank] + r * a.row_bytes;
        } else {
            const int code = a.row_src[r - a.T];
            const int s = code >> kEpRankShift, t = code & kEpRowMask;
            if (s < 0 || s >= a.world || t >= a.T) {    // never written so by ep_rows_kernel
                if (lane == 0) atomicOr(a.status, MOK_STATUS_BAD_INDEX);
                continue;
            }
            src = a.src[s] + t * a.row_bytes;
        }
        const V *sv = reinterpret_cast<const V *>(src);
        V *dv = reinterpret_cast<V *>(a.dst + r * a.row_bytes);
        for (int c = lane; c < vec; c += 128) {
            V q[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c + 32 * u < vec) q[u] = sv[c + 32 * u];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (c + 32 * u < vec) dv[c + 32 * u] = q[u];
        }
    }
}

template <typename V>
__global__ void __launch_bounds__(256) ep_pull_kernel(EpPull a)
{
    ep_pull_rows<V>(a, (blockIdx.x * blockDim.x + threadIdx.x) >> 5, (gridDim.x * blockDim.x) >> 5, threadIdx.x & 31);
}

// MXFP8 training, owner side, over its own and received rows (T + *n_recv, H
// wide): quantise the pulled bf16 dy rows into e4m3 codes and row-major ue8m0
// scales (the MXFP8 down dgrad's operand; a row's 1x32 blocks depend on that row
// alone, so they equal the token's rank's own quantisation), and decode the
// pulled x codes into bf16 (the gate/up weight gradient's operand, exactly the
// values the forward used).  One 32-element block per thread and step.
struct EpMxPrep {
    const __nv_bfloat16 *dy;       // [rows, H] pulled dy rows
    uint8_t *dyq, *dys;            // [rows, H], [rows, H / 32]
    const uint8_t *xq, *xs;        // [rows, H], [rows, H / 32] pulled x codes and scales
    __nv_bfloat16 *xdq;            // [rows, H] decoded x
    const int *n_recv;
    int T, world, H;
};

__device__ __forceinline__ void ep_mx_prepare(const EpMxPrep &a, long long first, long long stride)
{
    const long long kb32 = a.H / 32;
    const long long nb = (a.T + min(*a.n_recv, a.world * a.T)) * kb32;
    for (long long b = first; b < nb; b += stride) {
        quantize_block(b, a.dy, a.dyq, a.dys, kb32, 0);
        const int e = static_cast<int>(a.xs[b]) - 127;
        const uint4 *q = reinterpret_cast<const uint4 *>(a.xq + b * 32);
        uint32_t w[8];
        const uint4 q0 = q[0], q1 = q[1];
        w[0] = q0.x; w[1] = q0.y; w[2] = q0.z; w[3] = q0.w; w[4] = q1.x; w[5] = q1.y; w[6] = q1.z; w[7] = q1.w;
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            p[i] = pack_bf16x2(mx_decode(w[i >> 1] >> (16 * (i & 1)), e), mx_decode(w[i >> 1] >> (16 * (i & 1) + 8), e));
        uint4 *d = reinterpret_cast<uint4 *>(a.xdq + b * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
    }
}

__global__ void __launch_bounds__(256) ep_mx_prepare_kernel(EpMxPrep a)
{
    ep_mx_prepare(a, blockIdx.x * 256ll + threadIdx.x, static_cast<long long>(gridDim.x) * 256);
}

// Per-rank pointer table in device memory (the push epilogues read it).
struct EpTable {
    float *p[kEpMaxRanks];
};
__global__ void ep_table_kernel(EpTable t, float **dst, int n)
{
    if (threadIdx.x < n) dst[threadIdx.x] = t.p[threadIdx.x];
}

// Backward: the slot-gradient partials <dy W_down, h> of every routed row the
// owner computed (nt floats per row, its down dgrad's N tiles) go to the row's
// source rank, at the row's position in the source's sorted rows, where the
// slot gradients are formed.  One thread per (row, tile).
__device__ __forceinline__ void ep_push_gpart(const float *gpart, const int *row_gdst, const int *seg, int n_seg,
                                              int nt, float *const *gdst, int world, int tk, int *status,
                                              long long first, long long stride)
{
    const long long n = static_cast<long long>(seg[n_seg]) * nt;
    for (long long i = first; i < n; i += stride) {
        const int r = static_cast<int>(i / nt), j = static_cast<int>(i - static_cast<long long>(r) * nt);
        const int code = row_gdst[r];
        const int s = code >> kEpRankShift, q = code & kEpRowMask;
        if (s < 0 || s >= world || q >= tk) {       // never written so by ep_rows_kernel
            atomicOr(status, MOK_STATUS_BAD_INDEX);
            continue;
        }
        gdst[s][static_cast<size_t>(q) * nt + j] = gpart[i];
    }
}

__global__ void __launch_bounds__(256) ep_push_gpart_kernel(const float *gpart, const int *row_gdst, const int *seg,
                                                            int n_seg, int nt, float **gdst, int world, int tk,
                                                            int *status)
{
    ep_push_gpart(gpart, row_gdst, seg, n_seg, nt, gdst, world, tk, status, blockIdx.x * 256ll + threadIdx.x,
                  static_cast<long long>(gridDim.x) * 256);
}

}  // namespace mok
