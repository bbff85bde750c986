// quant.cu -- the run-time quantizers: NVFP4 block-16 activation quantizer, fp8r
// per-row quantizer, the global-scale (amax) helper and the scale re-layout helper.
//
// "BFL (fp8r / nvfp4)" (Diffusers quantization doc): nvfp4 format bullet (E2M1
// packed two per byte, E4M3 scale per 16-element block, fp32 global scales) and
// fp8r bullet (activations quantized to E4M3 per row at run time); Kernels table
// (the nvfp4 path quantizes activations before the FP4 GEMM).
//
// Both quantizers are HBM-bound streaming kernels: 128-bit coalesced loads of bf16,
// warp-shuffle reductions, and coalesced stores of the packed codes.  The
// arithmetic is fixed step by step (IEEE binary32, round to nearest even, no FTZ,
// no fast-math) so that codes and scale bytes are bit-identical to the definition:
//   nvfp4: t = 6g ; s = t > 0 ? amax/t : 0 ; sb = E4M3(s) ; d = dec(sb)*g ;
//          d == 0 -> codes 0 ; else code = E2M1(x * min(1/d, FLT_MAX))
//   fp8r : s = amax/448 ; s == 0 -> codes 0 ; else q = E4M3(x * min(1/s, FLT_MAX))
#include <atomic>
#include <cfloat>
#include <cstdint>
#include <mutex>

#include "bsp_internal.h"
#include "bsp_testing.h"
#include "bsp_ptx.cuh"
#include "nvfp4_block.cuh"

namespace bsp {
namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const uint4* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8])
{
    f[0] = bf16lo_to_f32(v.x); f[1] = bf16hi_to_f32(v.x);
    f[2] = bf16lo_to_f32(v.y); f[3] = bf16hi_to_f32(v.y);
    f[4] = bf16lo_to_f32(v.z); f[5] = bf16hi_to_f32(v.z);
    f[6] = bf16lo_to_f32(v.w); f[7] = bf16hi_to_f32(v.w);
}

// Each thread owns whole 16-element blocks (two 16-byte loads), two blocks per
// iteration (block indices i and i + 32 within a 64-block warp span), with the next
// iteration's loads issued before the current blocks are encoded.  Lanes 4j..4j+3 of
// a warp hold 4 consecutive blocks of one row (K % 64 == 0 for the MMA layout), so the
// 4 scale bytes are gathered by shuffles and written as one word.
constexpr int kQBlocksPerWarp = 64;

struct Block16 {
    uint4 lo, hi;
};

__device__ __forceinline__ Block16 load_block(const uint4* x, int64_t blk, int64_t nblk)
{
    Block16 b;
    if (blk < nblk) {
        b.lo = ld_stream(x + 2 * blk);
        b.hi = ld_stream(x + 2 * blk + 1);
    } else {
        b.lo = make_uint4(0, 0, 0, 0);
        b.hi = b.lo;
    }
    return b;
}

// Encode one block of 16 bf16 (two 16-byte loads): see nvfp4_encode_block16.
__device__ __forceinline__ uint2 encode_block(const Block16& b, float g, float t, uint32_t& sb)
{
    const uint32_t v[8] = {b.lo.x, b.lo.y, b.lo.z, b.lo.w, b.hi.x, b.hi.y, b.hi.z, b.hi.w};
    return nvfp4_encode_block16(v, g, t, sb);
}

// Division by the blocks per row, n / d for 0 <= n < 2^31, as a multiply-high and a
// shift (round-up method: with 2^(l-1) < d <= 2^l and m = ceil(2^(31+l) / d), m < 2^32
// and floor(n*m / 2^(31+l)) = floor(n / d) for every such n).  m == 0 encodes d == 1.
struct RowDiv {
    uint32_t m, s;
};

RowDiv row_div(uint32_t d)
{
    RowDiv r{0, 0};
    if (d <= 1) return r;
    uint32_t l = 0;
    while ((uint64_t{1} << l) < d) ++l;
    const unsigned __int128 num = static_cast<unsigned __int128>(1) << (31 + l);
    r.m = static_cast<uint32_t>((num + d - 1) / d);
    r.s = l - 1;
    return r;
}

__device__ __forceinline__ uint32_t div_rows(uint32_t n, RowDiv r)
{
    return r.m ? (__umulhi(n, r.m) >> r.s) : n;
}

template <int LAYOUT>
__device__ __forceinline__ void store_block(uint2* codes, uint8_t* scales, int64_t blk,
                                            int64_t nblk, int64_t nb_row, int64_t kb4, uint2 w,
                                            uint32_t sb, int lane, RowDiv rd, bool idx32)
{
    // gather 4 consecutive blocks' scale bytes into lane 4j
    const uint32_t s1 = __shfl_down_sync(0xffffffffu, sb, 1);
    const uint32_t s2 = __shfl_down_sync(0xffffffffu, sb, 2);
    const uint32_t s3 = __shfl_down_sync(0xffffffffu, sb, 3);
    if (blk < nblk) {
        codes[blk] = w;
        if ((lane & 3) == 0) {
            const uint32_t w4 = sb | (s1 << 8) | (s2 << 16) | (s3 << 24);
            int64_t off;
            if (LAYOUT == BSP_SF_LINEAR) {
                off = blk;                                   // [rows][K/16] is the block index
            } else {
                const int64_t row = idx32 ? static_cast<int64_t>(div_rows(static_cast<uint32_t>(blk), rd))
                                          : blk / nb_row;
                off = sf_mma_offset(row, blk - row * nb_row, kb4);
            }
            if (blk + 3 < nblk && (off & 3) == 0) {
                *reinterpret_cast<uint32_t*>(scales + off) = w4;
            } else {                                         // ragged tail of a linear layout
                for (int i = 0; i < 4 && blk + i < nblk; ++i)
                    scales[off + i] = static_cast<uint8_t>(w4 >> (8 * i));
            }
        }
    }
}

// The kernel's global scale g.  Static: the fp32 at gptr.  Dynamic (partials != null):
// the per-CTA maxima of |x| that amax_kernel left as fp32 bit patterns are reduced here by
// every CTA, g = amax / (448 * 6) (one binary32 division, as nvfp4_global_scale), and CTA 0
// publishes g at gout for the GEMM that follows.  Every thread of the CTA must call it.
__device__ __forceinline__ float resolve_global_scale(const float* gptr, const uint32_t* partials,
                                                      int npartials, float* gout)
{
    if (partials == nullptr) return __ldg(gptr);
    __shared__ uint32_t red[32];
    uint32_t m = 0;
    for (int i = threadIdx.x; i < npartials; i += blockDim.x) m = max(m, __ldg(partials + i));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0u;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
        if (threadIdx.x == 0) red[0] = m;
    }
    __syncthreads();
    const float g = __fdiv_rn(__uint_as_float(red[0]), 2688.0f);
    if (blockIdx.x == 0 && threadIdx.x == 0) *gout = g;
    return g;
}

template <int LAYOUT, bool IDX32>
__global__ void __launch_bounds__(kQuantThreads)
    nvfp4_quant_kernel(const uint4* __restrict__ x, int64_t nblk, int64_t nb_row, RowDiv rd,
                       const float* __restrict__ gptr, uint2* __restrict__ codes,
                       uint8_t* __restrict__ scales, const uint32_t* __restrict__ partials,
                       int npartials, float* gout)
{
    // a GEMM launched as this grid's programmatic dependent may start its prologue now;
    // it still waits for this grid to complete before reading the codes
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
    const int64_t kb4 = (nb_row + 3) >> 2;
    const int64_t step = nwarps * kQBlocksPerWarp;

    // the first span's loads go out before the global scale is read (or reduced), so
    // their latency and that of g overlap instead of adding up
    int64_t base = warp * kQBlocksPerWarp;
    Block16 b0 = load_block(x, base + lane, nblk);
    Block16 b1 = load_block(x, base + 32 + lane, nblk);
    const float g = resolve_global_scale(gptr, partials, npartials, gout);
    const float t = __fmul_rn(6.0f, g);
    while (base < nblk) {
        const int64_t next = base + step;
        // prefetch the next span before encoding this one
        Block16 n0 = load_block(x, next + lane, nblk);
        Block16 n1 = load_block(x, next + 32 + lane, nblk);
        uint32_t sb0, sb1;
        const uint2 w0 = encode_block(b0, g, t, sb0);
        store_block<LAYOUT>(codes, scales, base + lane, nblk, nb_row, kb4, w0, sb0, lane, rd, IDX32);
        const uint2 w1 = encode_block(b1, g, t, sb1);
        store_block<LAYOUT>(codes, scales, base + 32 + lane, nblk, nb_row, kb4, w1, sb1, lane, rd,
                            IDX32);
        b0 = n0;
        b1 = n1;
        base = next;
    }
}

// Staged variant: one persistent CTA per SM streams a contiguous range of blocks through
// a ring of shared-memory chunks filled by bulk asynchronous copies (one thread issues
// them), so a whole chunk (62 KB) per stage is in flight instead of 64 bytes per thread;
// 31 consumer warps encode from shared memory exactly as above (same lane <-> block map,
// same stores).  All waits are bounded.
constexpr int kStageThreads = 1024;
constexpr int kStageWarps = kStageThreads / 32 - 1;              // consumer warps
constexpr int kChunkBlocks = kStageWarps * kQBlocksPerWarp;      // 1984 blocks
constexpr int kChunkBytes = kChunkBlocks * 32;                   // 62 KB of bf16
constexpr int kStageRing = 3;
constexpr int kStageSmem = kStageRing * kChunkBytes + 2 * kStageRing * 8 + 128;

__device__ __forceinline__ uint4 lds128(const uint8_t* p)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

template <int LAYOUT, bool IDX32>
__global__ void __launch_bounds__(kStageThreads, 1)
    nvfp4_quant_staged_kernel(const uint8_t* __restrict__ x, int64_t nblk, int64_t nb_row,
                              RowDiv rd, const float* __restrict__ gptr, uint2* __restrict__ codes,
                              uint8_t* __restrict__ scales, int64_t blocks_per_cta, int* status,
                              uint64_t wait_ns, const uint32_t* __restrict__ partials,
                              int npartials, float* gout)
{
    // a GEMM launched as this grid's programmatic dependent may start its prologue now;
    // it still waits for this grid to complete before reading the codes
    griddep_launch_dependents();
    const float g_cta = resolve_global_scale(gptr, partials, npartials, gout);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) &
                                               ~uintptr_t(127));
    uint64_t* full = reinterpret_cast<uint64_t*>(ring + kStageRing * kChunkBytes);
    uint64_t* empty = full + kStageRing;
    __shared__ int abort_word;
    volatile int* abort_flag = &abort_word;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kStageRing; ++i) {
            mbar_init(full + i, 1);
            mbar_init(empty + i, kStageWarps);
        }
        abort_word = 0;
        fence_mbar_init();
    }
    __syncthreads();
    const int64_t b0 = static_cast<int64_t>(blockIdx.x) * blocks_per_cta;
    const int64_t b1 = b0 + blocks_per_cta < nblk ? b0 + blocks_per_cta : nblk;
    const int64_t nchunks = b1 > b0 ? (b1 - b0 + kChunkBlocks - 1) / kChunkBlocks : 0;
    if (warp == 0) {
        if (lane == 0) {
            int64_t i = 0;
            for (; i < nchunks; ++i) {
                const int st = static_cast<int>(i % kStageRing);
                const uint32_t ph = static_cast<uint32_t>((i / kStageRing) & 1);
                if (i >= kStageRing &&
                    !mbar_wait(empty + st, ph ^ 1u, abort_flag, wait_ns, status, 31))
                    break;
                const int64_t c = b0 + i * kChunkBlocks;
                const int64_t nb = b1 - c < kChunkBlocks ? b1 - c : kChunkBlocks;
                const uint32_t bytes = static_cast<uint32_t>(nb * 32);
                mbar_arrive_expect_tx(full + st, bytes);
                bulk_load(ring + st * kChunkBytes, x + c * 32, bytes, full + st);
            }
            // every copy into the ring lands before the CTA may exit (abort path)
            for (int64_t j = (i > kStageRing ? i - kStageRing : 0); j < i; ++j)
                drain_wait(full + (j % kStageRing), static_cast<uint32_t>((j / kStageRing) & 1),
                           wait_ns, status);
        }
    } else {
        const float g = g_cta;
        const float t = __fmul_rn(6.0f, g);
        const int64_t kb4 = (nb_row + 3) >> 2;
        const int cw = warp - 1;
        for (int64_t i = 0; i < nchunks; ++i) {
            const int st = static_cast<int>(i % kStageRing);
            const uint32_t ph = static_cast<uint32_t>((i / kStageRing) & 1);
            const bool ok = mbar_wait(full + st, ph, abort_flag, wait_ns, status, 32);
            if (!__all_sync(0xffffffffu, ok)) break;
            const int64_t c = b0 + i * kChunkBlocks;
            const int64_t lim = b1 - c < kChunkBlocks ? b1 : c + kChunkBlocks;   // chunk end
            const uint8_t* src = ring + st * kChunkBytes + cw * kQBlocksPerWarp * 32;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t blk = c + cw * kQBlocksPerWarp + h * 32 + lane;
                Block16 b;
                if (blk < lim) {
                    b.lo = lds128(src + (h * 32 + lane) * 32);
                    b.hi = lds128(src + (h * 32 + lane) * 32 + 16);
                } else {
                    b.lo = make_uint4(0, 0, 0, 0);
                    b.hi = b.lo;
                }
                uint32_t sb;
                const uint2 w = encode_block(b, g, t, sb);
                store_block<LAYOUT>(codes, scales, blk, lim, nb_row, kb4, w, sb, lane, rd, IDX32);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + st);
        }
    }
}

// ---------------------------------------------------------------- fp8r
constexpr int kRowThreads = 128;

__device__ __forceinline__ float block_max_128(float v, float* red)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    v = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    return v;
}

__device__ __forceinline__ uint2 quant8_e4m3(const float (&f)[8], float r)
{
    uint2 q;
    q.x = cvt_e4m3x2(__fmul_rn(f[0], r), __fmul_rn(f[1], r)) |
          (cvt_e4m3x2(__fmul_rn(f[2], r), __fmul_rn(f[3], r)) << 16);
    q.y = cvt_e4m3x2(__fmul_rn(f[4], r), __fmul_rn(f[5], r)) |
          (cvt_e4m3x2(__fmul_rn(f[6], r), __fmul_rn(f[7], r)) << 16);
    return q;
}

// One CTA per row; the row is held in registers (CPT chunks of 8 per thread).
template <int CPT>
__global__ void __launch_bounds__(kRowThreads)
    fp8r_quant_kernel(const uint4* __restrict__ x, int64_t K8, uint2* __restrict__ q,
                      float* __restrict__ row_scale)
{
    __shared__ float red[4];
    const int64_t row = blockIdx.x;
    const uint4* xr = x + row * K8;
    uint2* qr = q + row * K8;
    uint4 v[CPT];
    float amax = 0.0f;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int64_t i = threadIdx.x + c * kRowThreads;
        v[c] = (i < K8) ? ld_stream(xr + i) : make_uint4(0, 0, 0, 0);
        float f[8];
        unpack8(v[c], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
    }
    amax = block_max_128(amax, red);
    const float s = __fdiv_rn(amax, 448.0f);
    if (threadIdx.x == 0) row_scale[row] = s;
    const float r = (s == 0.0f) ? 0.0f : fminf(__frcp_rn(s), FLT_MAX);
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int64_t i = threadIdx.x + c * kRowThreads;
        if (i < K8) {
            float f[8];
            unpack8(v[c], f);
            qr[i] = (s == 0.0f) ? make_uint2(0, 0) : quant8_e4m3(f, r);
        }
    }
}

// Rows too long to hold on chip: two passes over the row.
__global__ void __launch_bounds__(kRowThreads)
    fp8r_quant_long_kernel(const uint4* __restrict__ x, int64_t K8, uint2* __restrict__ q,
                           float* __restrict__ row_scale)
{
    __shared__ float red[4];
    const int64_t row = blockIdx.x;
    const uint4* xr = x + row * K8;
    uint2* qr = q + row * K8;
    float amax = 0.0f;
    for (int64_t i = threadIdx.x; i < K8; i += kRowThreads) {
        float f[8];
        unpack8(ld_stream(xr + i), f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
    }
    amax = block_max_128(amax, red);
    const float s = __fdiv_rn(amax, 448.0f);
    if (threadIdx.x == 0) row_scale[row] = s;
    const float r = (s == 0.0f) ? 0.0f : fminf(__frcp_rn(s), FLT_MAX);
    for (int64_t i = threadIdx.x; i < K8; i += kRowThreads) {
        float f[8];
        unpack8(ld_stream(xr + i), f);
        qr[i] = (s == 0.0f) ? make_uint2(0, 0) : quant8_e4m3(f, r);
    }
}

// ---------------------------------------------------------------- global scale
// amax(|x|) over bf16 values, as the bit pattern of a non-negative fp32 (atomic max on
// *out, which the caller clears first).  Each thread keeps four 16-byte loads in flight
// and takes the max on the sign-cleared bf16 bit patterns (max.bf16x2, starting from 0 so
// a NaN loses as with fmaxf); the largest |x| is exact in bf16, so the result is the
// binary32 max of |x|.
template <bool PARTIAL>
__global__ void __launch_bounds__(256)
    amax_kernel(const uint4* __restrict__ x, int64_t n8, unsigned int* __restrict__ out)
{
    __shared__ uint32_t red[8];
    uint32_t m2 = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * 256;
    int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    for (; i + 3 * stride < n8; i += 4 * stride) {
        uint4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = ld_stream(x + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            m2 = max_bf16x2(m2, v[u].x & 0x7FFF7FFFu);
            m2 = max_bf16x2(m2, v[u].y & 0x7FFF7FFFu);
            m2 = max_bf16x2(m2, v[u].z & 0x7FFF7FFFu);
            m2 = max_bf16x2(m2, v[u].w & 0x7FFF7FFFu);
        }
    }
    for (; i < n8; i += stride) {
        const uint4 v = ld_stream(x + i);
        m2 = max_bf16x2(m2, v.x & 0x7FFF7FFFu);
        m2 = max_bf16x2(m2, v.y & 0x7FFF7FFFu);
        m2 = max_bf16x2(m2, v.z & 0x7FFF7FFFu);
        m2 = max_bf16x2(m2, v.w & 0x7FFF7FFFu);
    }
    m2 = max_bf16x2(m2, __byte_perm(m2, 0, 0x1032));
    uint32_t m = m2 << 16;                       // fp32 bits of the larger |x|
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = red[0];
        for (int w = 1; w < 8; ++w) b = max(b, red[w]);
        // non-negative floats order like their bit patterns
        if (PARTIAL)
            out[blockIdx.x] = b;           // one slot per CTA, reduced by the quantizer
        else
            atomicMax(out, b);
    }
}

__global__ void global_scale_finalize_kernel(float* out)
{
    const float amax = __uint_as_float(*reinterpret_cast<unsigned int*>(out));
    out[0] = __fdiv_rn(amax, 2688.0f);
}

// ---------------------------------------------------------------- scale re-layout
__global__ void sf_to_mma_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                 int64_t rows, int64_t nb, int64_t kb4, int64_t dst_bytes)
{
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < dst_bytes;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t tile = j >> 9, within = j & 511;
        const int64_t rt = tile / kb4, ct = tile - rt * kb4;
        const int64_t row = rt * 128 + ((within & 15) >> 2) * 32 + (within >> 4);
        const int64_t kb = ct * 4 + (within & 3);
        dst[j] = (row < rows && kb < nb) ? src[row * nb + kb] : 0;
    }
}

__global__ void sf_to_linear_kernel(const uint8_t* __restrict__ src, uint8_t* __restrict__ dst,
                                    int64_t rows, int64_t nb, int64_t kb4)
{
    const int64_t n = rows * nb;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t row = j / nb, kb = j - row * nb;
        dst[j] = src[sf_mma_offset(row, kb, kb4)];
    }
}

// NVFP4 -> bf16 decode (the dequantise-only fallback's weight decode): one thread per
// 16-element block.  Per element, in binary32 with round to nearest even:
// p = e2m1(code) * e4m3(sb) (exact), y = p * g, then one rounding to bf16.
__device__ __forceinline__ void e2m1x2_to_f32(uint32_t byte, float& lo, float& hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 c;\n\tcvt.u8.u32 c, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, c;\n\t}"
        : "=r"(h2)
        : "r"(byte));
    // element 2j sits in the low nibble and comes out in the low half
    lo = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
    hi = __half2float(__ushort_as_half(static_cast<unsigned short>(h2 >> 16)));
}

template <int LAYOUT>
__global__ void __launch_bounds__(256)
    nvfp4_dequant_kernel(const uint32_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                         const float* __restrict__ gptr, uint4* __restrict__ out, int64_t nhalf,
                         int64_t nb_row)
{
    // one thread per half block (8 elements): 4 code bytes in, 16 bytes of bf16 out, so a
    // warp's loads and stores are both contiguous
    griddep_launch_dependents();
    const float g = __ldg(gptr);
    const int64_t kb4 = (nb_row + 3) >> 2;
    for (int64_t h = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; h < nhalf;
         h += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const uint32_t c = __ldg(codes + h);
        const int64_t blk = h >> 1;
        int64_t off;
        if (LAYOUT == BSP_SF_LINEAR) {
            off = blk;
        } else {
            const int64_t row = blk / nb_row;
            off = sf_mma_offset(row, blk - row * nb_row, kb4);
        }
        const float sd = e4m3_to_f32(__ldg(scales + off));
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float lo, hi;
            e2m1x2_to_f32((c >> (8 * j)) & 0xFFu, lo, hi);
            lo = __fmul_rn(__fmul_rn(lo, sd), g);
            hi = __fmul_rn(__fmul_rn(hi, sd), g);
            __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
            w[j] = *reinterpret_cast<uint32_t*>(&b);
        }
        out[h] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// NVFP4 quantizer kernel choice: 0 = by size, 1 = grid-stride, 2 = staged (test hook)
std::atomic<int> g_quant_choice{0};

int quant_kernel_choice() { return g_quant_choice.load(); }

// Test hook kernel: the quantizers' conversions (cvt.rn.satfinite.e2m1x2.f32 /
// .e4m3x2.f32, through the same wrappers) applied to every fp32 whose bit pattern lies
// in [first, first + n).
__global__ void cvt_range_kernel(int kind, uint32_t first, int64_t n, uint8_t* __restrict__ out)
{
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float y = __uint_as_float(first + static_cast<uint32_t>(i));
        out[i] = static_cast<uint8_t>(kind == 0 ? (cvt_e2m1x2(y, 0.0f) & 0xFu)
                                                : (cvt_e4m3x2(y, 0.0f) & 0xFFu));
    }
}

int grid_for(int64_t work_items, int per_block, int num_sms, int blocks_per_sm)
{
    int64_t need = (work_items + per_block - 1) / per_block;
    int64_t cap = static_cast<int64_t>(num_sms) * blocks_per_sm;
    if (need < 1) need = 1;
    return static_cast<int>(need < cap ? need : cap);
}

}  // namespace
}  // namespace bsp

extern "C" {

int nvfp4_quantize_act(const void* x_bf16, int64_t M, int64_t K, const float* global_scale,
                       uint8_t* codes, uint8_t* scales, int layout, bsp_stream_t stream)
{
    return bsp::quantize_act_impl(x_bf16, M, K, global_scale, codes, scales, layout, stream,
                                  nullptr, 0, nullptr);
}

}  // extern "C"

namespace bsp {

int quantize_act_impl(const void* x_bf16, int64_t M, int64_t K, const float* global_scale,
                      uint8_t* codes, uint8_t* scales, int layout, bsp_stream_t stream,
                      const uint32_t* partials, int npartials, float* gout)
{
    if (M < 0 || K <= 0 || (layout != BSP_SF_LINEAR && layout != BSP_SF_MMA))
        return BSP_ERR_INVALID_ARG;
    if (M == 0) return BSP_OK;
    if (!x_bf16 || !global_scale || !codes || !scales) return BSP_ERR_INVALID_ARG;
    if (K % 16 != 0 || (layout == BSP_SF_MMA && K % 64 != 0)) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(codes) || !aligned16(scales) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u))
        return BSP_ERR_MISALIGNED;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    const int64_t nblk = M * (K / 16);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const RowDiv rd = row_div(static_cast<uint32_t>(K / 16));
    const int choice = quant_kernel_choice();
    // Large inputs: the staged kernel (bulk copies into a shared-memory ring, 85 % of HBM at
    // 65536 x 3072); below ~96 M elements the grid-stride kernel finishes sooner (its CTAs
    // start encoding after one 64-byte load instead of a 62 KB chunk).
    const bool staged = choice == 2 || (choice == 0 && nblk * 16 >= (int64_t{96} << 20));
    if (!staged) {
        // at most the resident grid (4 CTAs of 256 threads per SM at 64 registers)
        const int grid = grid_for(nblk, (kQuantThreads / 32) * kQBlocksPerWarp, sms, 4);
        const auto* xv = static_cast<const uint4*>(x_bf16);
        auto* cv = reinterpret_cast<uint2*>(codes);
        // 32-bit block indices (row by multiply-high) whenever a warp span past the end
        // still fits; the linear layout needs no row at all
        const bool idx32 =
            nblk + static_cast<int64_t>(grid) * kQuantThreads * 2 < (int64_t{1} << 31);
        if (layout == BSP_SF_LINEAR)
            nvfp4_quant_kernel<BSP_SF_LINEAR, false><<<grid, kQuantThreads, 0, s>>>(
                xv, nblk, K / 16, rd, global_scale, cv, scales, partials, npartials, gout);
        else if (idx32)
            nvfp4_quant_kernel<BSP_SF_MMA, true><<<grid, kQuantThreads, 0, s>>>(
                xv, nblk, K / 16, rd, global_scale, cv, scales, partials, npartials, gout);
        else
            nvfp4_quant_kernel<BSP_SF_MMA, false><<<grid, kQuantThreads, 0, s>>>(
                xv, nblk, K / 16, rd, global_scale, cv, scales, partials, npartials, gout);
        return launch_status();
    }
    // one persistent CTA per SM, each a contiguous range of whole 64-block warp spans
    static std::once_flag attr_once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    std::call_once(attr_once[dev], [dev] {
        cudaError_t e = cudaSuccess;
        for (auto k : {nvfp4_quant_staged_kernel<BSP_SF_LINEAR, false>,
                       nvfp4_quant_staged_kernel<BSP_SF_MMA, true>,
                       nvfp4_quant_staged_kernel<BSP_SF_MMA, false>})
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kStageSmem);
        if (e != cudaSuccess) cudaGetLastError();   // no stale error left behind
        attr_err[dev] = e;
    });
    if (attr_err[dev] != cudaSuccess) return BSP_ERR_CUDA;
    const int64_t spans = (nblk + kQBlocksPerWarp - 1) / kQBlocksPerWarp;
    const int64_t spans_per_cta = (spans + sms - 1) / sms;
    const int64_t bpc = spans_per_cta * kQBlocksPerWarp;
    const int grid = static_cast<int>((nblk + bpc - 1) / bpc);
    const auto* xb = static_cast<const uint8_t*>(x_bf16);
    auto* cv = reinterpret_cast<uint2*>(codes);
    const bool idx32 = nblk < (int64_t{1} << 31) - kChunkBlocks;
    int* status = device_status_ptr(dev);
    const uint64_t wns = wait_limit_ns();
    if (layout == BSP_SF_LINEAR)
        nvfp4_quant_staged_kernel<BSP_SF_LINEAR, false><<<grid, kStageThreads, kStageSmem, s>>>(
            xb, nblk, K / 16, rd, global_scale, cv, scales, bpc, status, wns, partials,
            npartials, gout);
    else if (idx32)
        nvfp4_quant_staged_kernel<BSP_SF_MMA, true><<<grid, kStageThreads, kStageSmem, s>>>(
            xb, nblk, K / 16, rd, global_scale, cv, scales, bpc, status, wns, partials,
            npartials, gout);
    else
        nvfp4_quant_staged_kernel<BSP_SF_MMA, false><<<grid, kStageThreads, kStageSmem, s>>>(
            xb, nblk, K / 16, rd, global_scale, cv, scales, bpc, status, wns, partials,
            npartials, gout);
    return launch_status();
}

// The nvfp4 front half of a linear with a per-call activation scale: per-CTA maxima of |x|
// into `partials` (at most kDynamicPartials slots), then the quantizer, whose CTAs reduce
// them to g = amax / (448 * 6) and publish g at `g_out`.  Two launches, no clear.
int dynamic_quantize_front(const void* x_bf16, int64_t M, int64_t K, uint32_t* partials,
                           float* g_out, uint8_t* codes, uint8_t* scales, bsp_stream_t stream)
{
    if (M <= 0 || K <= 0 || K % 64 != 0 || !x_bf16 || !partials || !g_out) return BSP_ERR_INVALID_ARG;
    if (!aligned16(x_bf16)) return BSP_ERR_MISALIGNED;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    const int64_t n8 = M * K / 8;
    int grid = grid_for(n8, 256 * 4, sms, 8);
    if (grid > kDynamicPartials) grid = kDynamicPartials;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    amax_kernel<true><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x_bf16), n8, partials);
    st = launch_status();
    if (st != BSP_OK) return st;
    return quantize_act_impl(x_bf16, M, K, g_out, codes, scales, BSP_SF_MMA, stream, partials, grid,
                             g_out);
}

}  // namespace bsp

extern "C" {

int bsp_testing_cvt_range(int kind, uint32_t first, int64_t n, uint8_t* out, bsp_stream_t stream)
{
    using namespace bsp;
    if ((kind != 0 && kind != 1) || n < 0 || n > (int64_t{1} << 32) - first) return BSP_ERR_INVALID_ARG;
    if (n == 0) return BSP_OK;
    if (!out) return BSP_ERR_INVALID_ARG;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    const int grid = grid_for(n, 256 * 8, sms, 8);
    cvt_range_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(kind, first, n, out);
    return launch_status();
}

int bsp_testing_set_quant_kernel(int choice)
{
    if (choice < 0 || choice > 2) return BSP_ERR_INVALID_ARG;
    return bsp::g_quant_choice.exchange(choice);
}

int fp8r_quantize_rows(const void* x_bf16, int64_t M, int64_t K, uint8_t* q_e4m3,
                       float* row_scale, bsp_stream_t stream)
{
    using namespace bsp;
    if (M < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (M == 0) return BSP_OK;
    if (!x_bf16 || !q_e4m3 || !row_scale) return BSP_ERR_INVALID_ARG;
    if (K % 8 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (M > 0x7FFFFFFF) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || !aligned16(q_e4m3) || !aligned16(row_scale))
        return BSP_ERR_MISALIGNED;
    int st = check_device(nullptr, nullptr);
    if (st != BSP_OK) return st;
    const int64_t K8 = K / 8;
    const int64_t cpt = (K8 + kRowThreads - 1) / kRowThreads;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const auto* xv = static_cast<const uint4*>(x_bf16);
    auto* qv = reinterpret_cast<uint2*>(q_e4m3);
    const dim3 grid(static_cast<unsigned>(M));
    if (cpt <= 1)
        fp8r_quant_kernel<1><<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    else if (cpt <= 2)
        fp8r_quant_kernel<2><<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    else if (cpt <= 4)
        fp8r_quant_kernel<4><<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    else if (cpt <= 8)
        fp8r_quant_kernel<8><<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    else if (cpt <= 16)
        fp8r_quant_kernel<16><<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    else
        fp8r_quant_long_kernel<<<grid, kRowThreads, 0, s>>>(xv, K8, qv, row_scale);
    return launch_status();
}

int nvfp4_global_scale(const void* x_bf16, int64_t n, float* global_scale_out,
                       bsp_stream_t stream)
{
    using namespace bsp;
    if (n < 0 || !x_bf16 || !global_scale_out) return BSP_ERR_INVALID_ARG;
    if (n % 8 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x_bf16) || (reinterpret_cast<uintptr_t>(global_scale_out) & 3u))
        return BSP_ERR_MISALIGNED;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(global_scale_out, 0, sizeof(float), s) != cudaSuccess) {
        cudaGetLastError();
        return BSP_ERR_CUDA;
    }
    if (n > 0) {
        const int grid = grid_for(n / 8, 256 * 4, sms, 8);
        amax_kernel<false><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x_bf16), n / 8,
                                         reinterpret_cast<unsigned int*>(global_scale_out));
        st = launch_status();
        if (st != BSP_OK) return st;
    }
    global_scale_finalize_kernel<<<1, 1, 0, s>>>(global_scale_out);
    return launch_status();
}

int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, int layout,
                     const float* global_scale, int64_t rows, int64_t K, void* out_bf16,
                     bsp_stream_t stream)
{
    using namespace bsp;
    if (rows < 0 || K <= 0 || (layout != BSP_SF_LINEAR && layout != BSP_SF_MMA))
        return BSP_ERR_INVALID_ARG;
    if (rows == 0) return BSP_OK;
    if (!codes || !scales || !global_scale || !out_bf16) return BSP_ERR_INVALID_ARG;
    if (K % 16 != 0 || (layout == BSP_SF_MMA && K % 64 != 0)) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(codes) || !aligned16(out_bf16) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u))
        return BSP_ERR_MISALIGNED;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    const int64_t nhalf = rows * (K / 8);
    const int grid = grid_for(nhalf, 256 * 2, sms, 8);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const auto* cv = reinterpret_cast<const uint32_t*>(codes);
    auto* ov = static_cast<uint4*>(out_bf16);
    if (layout == BSP_SF_LINEAR)
        nvfp4_dequant_kernel<BSP_SF_LINEAR><<<grid, 256, 0, s>>>(cv, scales, global_scale, ov,
                                                                  nhalf, K / 16);
    else
        nvfp4_dequant_kernel<BSP_SF_MMA><<<grid, 256, 0, s>>>(cv, scales, global_scale, ov,
                                                               nhalf, K / 16);
    return launch_status();
}

int nvfp4_sf_convert(const uint8_t* src, uint8_t* dst, int64_t rows, int64_t K, int from,
                     int to, bsp_stream_t stream)
{
    using namespace bsp;
    if (rows < 0 || K <= 0) return BSP_ERR_INVALID_ARG;
    if (rows == 0) return BSP_OK;
    if (!src || !dst) return BSP_ERR_INVALID_ARG;
    if ((from != BSP_SF_LINEAR && from != BSP_SF_MMA) || (to != BSP_SF_LINEAR && to != BSP_SF_MMA) ||
        from == to)
        return BSP_ERR_INVALID_ARG;
    if (K % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    int dev = 0, sms = 0;
    int st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;
    const int64_t nb = K / 16, kb4 = (nb + 3) / 4;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (to == BSP_SF_MMA) {
        const int64_t bytes = nvfp4_sf_bytes(rows, K, BSP_SF_MMA);
        sf_to_mma_kernel<<<grid_for(bytes, 256, sms, 8), 256, 0, s>>>(src, dst, rows, nb, kb4,
                                                                       bytes);
    } else {
        sf_to_linear_kernel<<<grid_for(rows * nb, 256, sms, 8), 256, 0, s>>>(src, dst, rows, nb,
                                                                             kb4);
    }
    return launch_status();
}

}  // extern "C"
