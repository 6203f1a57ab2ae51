// quant.cuh -- MXFP8 quantisation (e4m3 elements, one ue8m0 scale per 32
// consecutive elements along the contraction axis), as used by the MXFP8
// forward ("Megakernels are dead and back…", section "Números de MoK").
//
// Block rule: e = smallest integer with amax <= 448 * 2^e (448 = largest e4m3
// value), clamped to [-127, 127], an all-zero block taking -127; the scale byte
// is e + 127 and every element is x * 2^-e rounded to nearest even e4m3 with
// saturation.  With this rule no element saturates.
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include "ptx.cuh"

namespace mok {

// Exponent of the block from the fp32 bit pattern of amax (exact integer logic):
// amax = (1 + f) 2^p; 448 * 2^(p-8) = 1.75 * 2^p covers it iff f <= 0.75.
__device__ __forceinline__ int mx_exponent(float amax)
{
    const uint32_t b = __float_as_uint(amax);
    const int biased = static_cast<int>(b >> 23);
    if (biased == 0) return -127;                    // zero or subnormal: far below 448 * 2^-127
    const int p = biased - 127;
    int e = p - 8 + ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    return max(-127, min(127, e));
}

__device__ __forceinline__ float exp2_neg(int e)   // 2^-e for e in [-127, 126]
{
    return __uint_as_float(static_cast<uint32_t>(127 - e) << 23);
}

// Thread = one block of 32 bf16 values: 64-byte load, 32-byte store.
// Byte offset of scale (row, j) (j = 32-element block along K) in the packed
// weight-scale layout: (K/128) x (rows/128) tiles of 512 bytes, tile (kb, rb)
// holding for row r = 128 rb + 32 q + i and block j = 4 kb + s the byte at
// 16 i + 4 q + s.  That is the layout the block-scaled MMA's scale-factor
// copy reads for a 128-row block, so one K block of a weight tile's scales
// is one contiguous 512-byte copy per 128 rows.
__device__ __forceinline__ long long packed_scale_offset(long long row, long long j, long long row_tiles)
{
    return ((j >> 2) * row_tiles + (row >> 7)) * 512 + (row & 31) * 16 + ((row >> 5) & 3) * 4 + (j & 3);
}

// e4m3 codes (4 per word, low byte first) of 32 values, scaled by 2^-e; two
// values per conversion (the pair's first value in the low byte)
__device__ __forceinline__ void mx_codes32(const float *v, int e, uint32_t *w)
{
    const float s = exp2_neg(e);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * s, v[4 * i + 1] * s), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * s, v[4 * i + 3] * s), __NV_SATFINITE, __NV_E4M3);
        w[i] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
}

// value of e4m3 code byte c times 2^e (exact; representable in bf16)
__device__ __forceinline__ float mx_decode(uint32_t c, int e)
{
    const __half_raw h = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c & 0xFFu), __NV_E4M3);
    return ldexpf(__half2float(__half(h)), e);
}

// Block b (32 elements) of src.  row_tiles = 0: scales [rows, K/32] row-major;
// row_tiles = rows / 128: packed layout.  deq (or null): the dequantised values
// in bf16 (exact), for the MXFP8 backward's weight gradient
__device__ __forceinline__ void quantize_block(long long b, const __nv_bfloat16 *__restrict__ src,
                                               uint8_t *__restrict__ q, uint8_t *__restrict__ scales, long long kb32,
                                               long long row_tiles, __nv_bfloat16 *__restrict__ deq = nullptr)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(src + b * 32);
    float v[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 u = p[i];
        v[8 * i + 0] = bf16_lo(u.x); v[8 * i + 1] = bf16_hi(u.x);
        v[8 * i + 2] = bf16_lo(u.y); v[8 * i + 3] = bf16_hi(u.y);
        v[8 * i + 4] = bf16_lo(u.z); v[8 * i + 5] = bf16_hi(u.z);
        v[8 * i + 6] = bf16_lo(u.w); v[8 * i + 7] = bf16_hi(u.w);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int e = mx_exponent(amax);
    uint32_t w[8];
    mx_codes32(v, e, w);
    uint4 *dst = reinterpret_cast<uint4 *>(q + b * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    const long long at = row_tiles ? packed_scale_offset(b / kb32, b % kb32, row_tiles) : b;
    scales[at] = static_cast<uint8_t>(e + 127);
    if (deq) {
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            p[i] = pack_bf16x2(mx_decode(w[i >> 1] >> (16 * (i & 1)), e), mx_decode(w[i >> 1] >> (16 * (i & 1) + 8), e));
        uint4 *d = reinterpret_cast<uint4 *>(deq + b * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) d[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
    }
}

__global__ void __launch_bounds__(256) quantize_mxfp8_kernel(const __nv_bfloat16 *__restrict__ src,
                                                             long long nblocks, uint8_t *__restrict__ q,
                                                             uint8_t *__restrict__ scales, long long kb32,
                                                             long long row_tiles, __nv_bfloat16 *__restrict__ deq)
{
    griddep_enter();
    const long long b = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (b < nblocks) quantize_block(b, src, q, scales, kb32, row_tiles, deq);
}

// Transposed quantisation: thread = (matrix b, column c, 32-row block j) of src
// [batch, R, C]; its 32 values down the column become row (b*C + c), K block j
// of q [batch*C, R], scale packed for that matrix (row_tiles = batch*C/128).
// Consecutive threads take consecutive columns, so each of the 32 row loads of
// a warp is one 64-byte segment.
__global__ void __launch_bounds__(256) quantize_mxfp8_t_kernel(const __nv_bfloat16 *__restrict__ src,
                                                               long long batch, long long R, long long C,
                                                               uint8_t *__restrict__ q, uint8_t *__restrict__ scales)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long kb32 = R / 32;
    if (i >= batch * C * kb32) return;
    const long long c = i % C, j = (i / C) % kb32, b = i / (C * kb32);
    const __nv_bfloat16 *col = src + (b * R + j * 32) * C + c;
    float v[32];
#pragma unroll
    for (int r = 0; r < 32; ++r) v[r] = __bfloat162float(col[r * C]);
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < 32; ++r) amax = fmaxf(amax, fabsf(v[r]));
    const int e = mx_exponent(amax);
    uint32_t w[8];
    mx_codes32(v, e, w);
    const long long row = b * C + c;
    uint4 *dst = reinterpret_cast<uint4 *>(q + row * R + j * 32);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    scales[packed_scale_offset(row, j, batch * C / 128)] = static_cast<uint8_t>(e + 127);
}


// Both MXFP8 copies of a weight tensor src [batch, R, C] from one read of it: the
// forward's (q [batch, R, C] along C, scales packed for [batch*R, C]) and the
// backward's (qt [batch, C, R] along R, scales packed for [batch*C, R]).  CTA =
// a 32 x 256 tile (32 rows of R, 256 columns of C) staged in shared memory;
// thread t then quantises row block (t % 32, t / 32) of the tile for q and column
// t for qt (a warp reads 32 rows, or 32 columns, so shared memory sees no bank
// conflict), with the arithmetic of quantize_block and quantize_mxfp8_t_kernel.
constexpr int kQuantBothCols = 256;
__global__ void __launch_bounds__(256) quantize_mxfp8_both_kernel(const __nv_bfloat16 *__restrict__ src,
                                                                  long long batch, long long R, long long C,
                                                                  uint8_t *__restrict__ q, uint8_t *__restrict__ s,
                                                                  uint8_t *__restrict__ qt,
                                                                  uint8_t *__restrict__ st)
{
    // bf16 tile; a row is 264 elements (132 words): the 32 rows of a warp's 16-byte
    // row reads fall on 8 distinct groups of 4 banks (4 wavefronts, the minimum)
    __shared__ __align__(16) __nv_bfloat16 tile[32][kQuantBothCols + 8];
    const long long ct = C / kQuantBothCols, rt = R / 32;
    const long long b = blockIdx.x / (ct * rt);
    const long long r0 = (blockIdx.x / ct) % rt * 32, c0 = blockIdx.x % ct * kQuantBothCols;
    const int t = threadIdx.x;
    // stage: 32 rows x 256 columns, 16-byte loads (a warp reads one 512-byte row piece)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int idx = i * 256 + t, row = idx >> 5, c8 = (idx & 31) * 8;
        *reinterpret_cast<uint4 *>(&tile[row][c8]) =
            *reinterpret_cast<const uint4 *>(src + ((b * R + r0 + row) * C + c0 + c8));
    }
    __syncthreads();
    float v[32];
    uint32_t w[8];
    {   // the forward's copy: 32 consecutive columns of one row
        const int row = t & 31, blk = t >> 5;
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 u = *reinterpret_cast<const uint4 *>(&tile[row][blk * 32 + 8 * i]);
            v[8 * i + 0] = bf16_lo(u.x); v[8 * i + 1] = bf16_hi(u.x); v[8 * i + 2] = bf16_lo(u.y);
            v[8 * i + 3] = bf16_hi(u.y); v[8 * i + 4] = bf16_lo(u.z); v[8 * i + 5] = bf16_hi(u.z);
            v[8 * i + 6] = bf16_lo(u.w); v[8 * i + 7] = bf16_hi(u.w);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
        const int e = mx_exponent(amax);
        mx_codes32(v, e, w);
        const long long grow = b * R + r0 + row, gcol = c0 + blk * 32;
        uint4 *dst = reinterpret_cast<uint4 *>(q + grow * C + gcol);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        s[packed_scale_offset(grow, gcol / 32, batch * R / 128)] = static_cast<uint8_t>(e + 127);
    }
    {   // the backward's copy: column t, 32 consecutive rows
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            v[i] = __bfloat162float(tile[i][t]);
            amax = fmaxf(amax, fabsf(v[i]));
        }
        const int e = mx_exponent(amax);
        mx_codes32(v, e, w);
        const long long grow = b * C + c0 + t;
        uint4 *dst = reinterpret_cast<uint4 *>(qt + grow * R + r0);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        st[packed_scale_offset(grow, r0 / 32, batch * C / 128)] = static_cast<uint8_t>(e + 127);
    }
}

}  // namespace mok
