// gemm.cu -- block-scaled GEMMs on the sm_100a tensor cores (tcgen05).
//
// "BFL (fp8r / nvfp4)" (Diffusers quantization doc), Kernels table: the nvfp4 linear
// runs a block-scaled FP4 GEMM on quantized activations and weights; the fp8r linear
// runs an FP8 GEMM with per-row scales.  Weights stay in their low-precision storage.
//
//   nvfp4: Y = bf16( acc * (a_global * w_global) + bias ),
//          acc = sum_k e2m1(a) e4m3(sa[k/16]) e2m1(w) e4m3(sw[k/16])  (tcgen05
//          kind::mxf4nvf4, block16 scale vectors, fp32 accumulation in TMEM)
//   fp8r : Y = bf16( (acc * sA[m]) * sW[n] + bias ), acc = sum_k e4m3(a) e4m3(w)
//          (tcgen05 kind::f8f6f4, fp32 accumulation in TMEM)
//
// Kernel design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: per K-stage, a 128x128-byte A tile and a BNx128-byte B
//               tile (128-byte swizzle) by cp.async.bulk.tensor, plus the scale-factor
//               blocks of both operands by plain bulk copies, all completing on the
//               stage's "full" mbarrier.
//   warp 1      allocates TMEM; one thread issues tcgen05.cp (scale factors smem ->
//               TMEM) and tcgen05.mma (4 per stage), then tcgen05.commit frees the
//               stage and, after the last stage, signals the accumulator.
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator (each warp reads its own
//               32-lane quadrant), scales, bias, bf16 rounding, stores.
// Tiles are 128 x BN; tile t of a CTA is blockIdx.x + i*gridDim.x, M-fastest so that
// neighbouring CTAs share the weight tile.  No cluster multicast is used anywhere.
#include <cfloat>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bsp_internal.h"
#include "bsp_ptx.cuh"
#include "bsp_testing.h"

namespace bsp {
namespace {

constexpr int kBM = 128;        // rows of A per tile (= TMEM lanes)
constexpr int kBKB = 128;       // bytes of K per stage and row (one 128-byte swizzle atom)
constexpr int kThreads = 192;   // 6 warps
constexpr uint32_t kTmemCols = 512;

struct GemmArgs {
    int M, N, K;                     // K in elements
    const uint8_t* sfa;              // nvfp4: MMA-layout block scales of A
    const uint8_t* sfb;              // nvfp4: MMA-layout block scales of W
    const float* a_scale;            // nvfp4: &input_scale ; fp8r: row scales of A [M]
    const float* w_scale;            // nvfp4: &weight_scale_2 ; fp8r: row scales of W [N]
    const __nv_bfloat16* bias;       // [N] or nullptr
    __nv_bfloat16* out;              // [M][N]
    int* status;                     // device status word
    uint64_t wait_ns;                // bounded-wait limit
    int64_t debug_stop_iter;         // < 0 in normal use; test hook, see bsp_testing.h
};

template <bool NVF4, int BN, int STAGES, int NACC>
struct Cfg {
    static constexpr int A_BYTES = kBM * kBKB;
    static constexpr int B_BYTES = BN * kBKB;
    static constexpr int SFA_BYTES = NVF4 ? 4 * 512 : 0;
    static constexpr int SFB_BYTES = NVF4 ? (BN / 128) * 4 * 512 : 0;
    static constexpr int K_STAGE = NVF4 ? 256 : 128;   // elements of K per stage
    static constexpr int K_MMA = NVF4 ? 64 : 32;       // elements of K per tcgen05.mma
    static constexpr int SFA_COL = NACC * BN;          // TMEM columns of the scale vectors
    static constexpr int SFB_COL = NACC * BN + 16;
    static constexpr int TMEM_USED = NACC * BN + (NVF4 ? 16 + 4 * (BN / 32) : 0);
    static constexpr int OFF_B = STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_BAR = OFF_SFB + STAGES * SFB_BYTES;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * NACC + 1;
    static constexpr int SMEM_BYTES = 1024 + OFF_BAR + NUM_BARS * 8 + 16;
    static constexpr uint32_t IDESC = NVF4 ? idesc_nvf4(kBM, BN) : idesc_e4m3(kBM, BN);
    static_assert(TMEM_USED <= (int)kTmemCols, "TMEM budget");
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(BN % 128 == 0 && BN <= 256, "tile width");
};

// Wait that ignores the abort flag (used on the way out, to drain work in flight).
__device__ __forceinline__ bool drain_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                           int* status)
{
    volatile int never = 0;
    return mbar_wait(bar, parity, &never, limit_ns, status, 90);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <bool NVF4, int BN, int STAGES, int NACC>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const GemmArgs args)
{
    using C = Cfg<NVF4, BN, STAGES, NACC>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::OFF_B;
    uint8_t* sSFA = smem + C::OFF_SFA;
    uint8_t* sSFB = smem + C::OFF_SFB;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* tfull = empty + STAGES;
    uint64_t* tempty = tfull + NACC;
    uint64_t* fin = tempty + NACC;
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(fin + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int M = args.M, N = args.N, K = args.K;
    const int num_m = (M + kBM - 1) / kBM;
    const int num_n = (N + BN - 1) / BN;
    const int num_tiles = num_m * num_n;
    const int num_kt = (K + C::K_STAGE - 1) / C::K_STAGE;
    const int kb4 = (K / 16 + 3) / 4;           // MMA-layout column tiles (nvfp4)
    const int num_n128 = (N + 127) / 128;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < NACC; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 4);
        }
        mbar_init(fin, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int64_t it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int mt = tile % num_m, nt = tile / num_m;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (it == args.debug_stop_iter) { ok = false; break; }
                    const int s = static_cast<int>(it % STAGES);
                    const uint32_t ph = static_cast<uint32_t>((it / STAGES) & 1);
                    if (!mbar_wait(empty + s, ph ^ 1u, abort_flag, args.wait_ns, args.status, 1)) {
                        ok = false;
                        break;
                    }
                    uint32_t bytes = C::A_BYTES + C::B_BYTES;
                    int nkb = 0, nvalid = 0;
                    if constexpr (NVF4) {
                        nkb = min(4, K / 64 - 4 * kt);
                        for (int c = 0; c < BN / 128; ++c)
                            nvalid += (nt * (BN / 128) + c < num_n128) ? 1 : 0;
                        bytes += static_cast<uint32_t>(nkb * 512 * (1 + nvalid));
                    }
                    mbar_arrive_expect_tx(full + s, bytes);
                    tma_load_2d(sA + s * C::A_BYTES, &tmA, full + s, kt * kBKB, mt * kBM);
                    tma_load_2d(sB + s * C::B_BYTES, &tmB, full + s, kt * kBKB, nt * BN);
                    if constexpr (NVF4) {
                        const int64_t a_off = (static_cast<int64_t>(mt) * kb4 + 4 * kt) * 512;
                        bulk_load(sSFA + s * C::SFA_BYTES, args.sfa + a_off, nkb * 512, full + s);
                        for (int c = 0; c < BN / 128; ++c) {
                            const int n128 = nt * (BN / 128) + c;
                            if (n128 < num_n128) {
                                const int64_t b_off =
                                    (static_cast<int64_t>(n128) * kb4 + 4 * kt) * 512;
                                bulk_load(sSFB + s * C::SFB_BYTES + c * 2048, args.sfb + b_off,
                                          nkb * 512, full + s);
                            }
                        }
                    }
                    ++it;
                }
            }
            // drain: the last STAGES loads issued must land before shared memory is freed
            for (int64_t i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
                drain_wait(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1),
                           args.wait_ns, args.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int64_t it = 0;
            int acc_it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                const int a = acc_it % NACC;
                const uint32_t aph = static_cast<uint32_t>((acc_it / NACC) & 1);
                if (!mbar_wait(tempty + a, aph ^ 1u, abort_flag, args.wait_ns, args.status, 2))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tbase + static_cast<uint32_t>(a * BN);
                for (int kt = 0; kt < num_kt; ++kt) {
                    const int s = static_cast<int>(it % STAGES);
                    const uint32_t ph = static_cast<uint32_t>((it / STAGES) & 1);
                    if (!mbar_wait(full + s, ph, abort_flag, args.wait_ns, args.status, 3)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    int nk;
                    if constexpr (NVF4) {
                        nk = min(4, K / 64 - 4 * kt);
                        for (int kb = 0; kb < nk; ++kb) {
                            tmem_cp_32x128b_x4(tbase + C::SFA_COL + kb * 4,
                                               sdesc_sf_block(smem_u32(sSFA + s * C::SFA_BYTES +
                                                                       kb * 512)));
#pragma unroll
                            for (int c = 0; c < BN / 128; ++c)
                                tmem_cp_32x128b_x4(
                                    tbase + C::SFB_COL + kb * (BN / 32) + c * 4,
                                    sdesc_sf_block(smem_u32(sSFB + s * C::SFB_BYTES + c * 2048 +
                                                            kb * 512)));
                        }
                    } else {
                        nk = min(4, (K - kt * C::K_STAGE + C::K_MMA - 1) / C::K_MMA);
                    }
                    const uint64_t adesc = sdesc_kmajor_sw128(smem_u32(sA + s * C::A_BYTES));
                    const uint64_t bdesc = sdesc_kmajor_sw128(smem_u32(sB + s * C::B_BYTES));
                    for (int k = 0; k < nk; ++k) {
                        // each MMA consumes 32 bytes of K: advance the start address by 2 x 16B
                        const uint32_t acc = (kt > 0 || k > 0) ? 1u : 0u;
                        if constexpr (NVF4)
                            mma_nvf4(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::IDESC,
                                     tbase + C::SFA_COL + k * 4, tbase + C::SFB_COL + k * (BN / 32),
                                     acc);
                        else
                            mma_f8f6f4(d_tmem, adesc + 2 * k, bdesc + 2 * k, C::IDESC, acc);
                    }
                    tc_commit(empty + s);
                    ++it;
                }
                if (!ok) break;
                tc_commit(tfull + a);
                ++acc_it;
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                 // TMEM lane quadrant of this warp
        const int row_in_tile = q * 32 + lane;
        float alpha = 0.0f;
        if constexpr (NVF4) alpha = __fmul_rn(__ldg(args.a_scale), __ldg(args.w_scale));
        int acc_it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mt = tile % num_m, nt = tile / num_m;
            const int a = acc_it % NACC;
            const uint32_t aph = static_cast<uint32_t>((acc_it / NACC) & 1);
            const bool ok = mbar_wait(tfull + a, aph, abort_flag, args.wait_ns, args.status, 4);
            if (!__all_sync(0xffffffffu, ok)) break;   // also reconverges the warp
            tc_fence_after();
            const int m = mt * kBM + row_in_tile;
            float sa = 0.0f;
            if constexpr (!NVF4) sa = (m < M) ? __ldg(args.a_scale + m) : 0.0f;
            const uint32_t taddr =
                tbase + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(a * BN);
            uint32_t packed[BN / 2];
#pragma unroll
            for (int j = 0; j < BN / 32; ++j) {
                uint32_t r[32];
                tmem_ld_x32(taddr + j * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int n = nt * BN + j * 32 + g * 8;   // 8-column group
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[g * 8 + i]);
                    if (n < N) {
                        if constexpr (NVF4) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(v[i], alpha);
                        } else {
                            const float4 w0 = __ldg(reinterpret_cast<const float4*>(args.w_scale + n));
                            const float4 w1 =
                                __ldg(reinterpret_cast<const float4*>(args.w_scale + n + 4));
                            const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(__fmul_rn(v[i], sa), sw[i]);
                        }
                        if (args.bias != nullptr) {
                            const uint4 b = __ldg(reinterpret_cast<const uint4*>(args.bias + n));
                            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                v[2 * i] = __fadd_rn(v[2 * i], bf16lo_to_f32(bw[i]));
                                v[2 * i + 1] = __fadd_rn(v[2 * i + 1], bf16hi_to_f32(bw[i]));
                            }
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        packed[j * 16 + g * 4 + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                }
            }
            // the accumulator is in registers now: hand TMEM back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + a);
            if (m < M) {
                __nv_bfloat16* orow = args.out + static_cast<int64_t>(m) * N;
#pragma unroll
                for (int j = 0; j < BN / 32; ++j)
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int n = nt * BN + j * 32 + g * 8;
                        if (n < N)
                            *reinterpret_cast<uint4*>(orow + n) =
                                make_uint4(packed[j * 16 + g * 4], packed[j * 16 + g * 4 + 1],
                                           packed[j * 16 + g * 4 + 2], packed[j * 16 + g * 4 + 3]);
                    }
            }
            ++acc_it;
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    if (warp == 1 && lane == 0) {
        tc_commit(fin);      // completes once every tcgen05 op of this thread is done
        drain_wait(fin, 0, args.wait_ns, args.status);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tbase, kTmemCols);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            cudaGetLastError();
    });
    return fn;
}

// 2-D byte tensor [rows][row_bytes], box of box_rows x 128 bytes, 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
             uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return BSP_ERR_CUDA;
    cuuint64_t dims[2] = {row_bytes, rows};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(kBKB), box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

template <bool NVF4, int BN, int STAGES, int NACC>
int launch(const uint8_t* a, const uint8_t* w, const GemmArgs& args, int dev, int sms,
           cudaStream_t s)
{
    using C = Cfg<NVF4, BN, STAGES, NACC>;
    static std::once_flag attr_once[64];
    static cudaError_t attr_err[64];
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(gemm_kernel<NVF4, BN, STAGES, NACC>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
    });
    if (attr_err[dev] != cudaSuccess) return BSP_ERR_CUDA;
    const uint64_t row_bytes = NVF4 ? static_cast<uint64_t>(args.K) / 2 : args.K;
    CUtensorMap tmA, tmB;
    int st = make_map(&tmA, a, row_bytes, static_cast<uint64_t>(args.M), kBM);
    if (st != BSP_OK) return st;
    st = make_map(&tmB, w, row_bytes, static_cast<uint64_t>(args.N), BN);
    if (st != BSP_OK) return st;
    const int64_t tiles =
        static_cast<int64_t>((args.M + kBM - 1) / kBM) * ((args.N + BN - 1) / BN);
    const int grid = static_cast<int>(tiles < sms ? tiles : sms);
    gemm_kernel<NVF4, BN, STAGES, NACC><<<grid, kThreads, C::SMEM_BYTES, s>>>(tmA, tmB, args);
    return launch_status();
}

int check_gemm_common(const void* a, const void* w, const void* bias, const void* out,
                      int64_t M, int64_t N, int64_t K)
{
    if (M < 0 || N < 0 || K < 0) return BSP_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return BSP_OK;
    if (!a || !w || !out) return BSP_ERR_INVALID_ARG;
    if (M > (1LL << 31) - 1 - kBM || N > (1LL << 31) - 1 - 256 || K > (1LL << 30))
        return BSP_ERR_UNSUPPORTED_SHAPE;
    if (N % 8 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(a) || !aligned16(w) || !aligned16(out) || (bias && !aligned16(bias)))
        return BSP_ERR_MISALIGNED;
    return BSP_OK;
}

int gemm_entry(bool nvf4, const uint8_t* a, const uint8_t* sfa, const float* a_scale,
               const uint8_t* w, const uint8_t* sfb, const float* w_scale, const void* bias,
               void* out, int64_t M, int64_t N, int64_t K, bsp_stream_t stream,
               int64_t debug_stop_iter, uint64_t wait_ns_override)
{
    int st = check_gemm_common(a, w, bias, out, M, N, K);
    if (st != BSP_OK || M == 0 || N == 0) return st;
    if (!a_scale || !w_scale) return BSP_ERR_INVALID_ARG;
    if (nvf4) {
        if (!sfa || !sfb) return BSP_ERR_INVALID_ARG;
        if (K < 64 || K % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(sfa) || !aligned16(sfb) || (reinterpret_cast<uintptr_t>(a_scale) & 3u) ||
            (reinterpret_cast<uintptr_t>(w_scale) & 3u))
            return BSP_ERR_MISALIGNED;
    } else {
        if (K < 16 || K % 16 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(a_scale) || !aligned16(w_scale)) return BSP_ERR_MISALIGNED;
    }
    int dev = 0, sms = 0;
    st = check_device(&dev, &sms);
    if (st != BSP_OK) return st;

    GemmArgs args;
    args.M = static_cast<int>(M);
    args.N = static_cast<int>(N);
    args.K = static_cast<int>(K);
    args.sfa = sfa;
    args.sfb = sfb;
    args.a_scale = a_scale;
    args.w_scale = w_scale;
    args.bias = static_cast<const __nv_bfloat16*>(bias);
    args.out = static_cast<__nv_bfloat16*>(out);
    args.status = device_status_ptr(dev);
    args.wait_ns = wait_ns_override ? wait_ns_override : wait_limit_ns();
    args.debug_stop_iter = debug_stop_iter;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (nvf4) {
        if (N > 128) return launch<true, 256, 4, 1>(a, w, args, dev, sms, s);
        return launch<true, 128, 6, 2>(a, w, args, dev, sms, s);
    }
    if (N > 128) return launch<false, 256, 4, 2>(a, w, args, dev, sms, s);
    return launch<false, 128, 6, 2>(a, w, args, dev, sms, s);
}

}  // namespace
}  // namespace bsp

extern "C" {

int nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
               const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
               const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
               bsp_stream_t stream)
{
    return bsp::gemm_entry(true, a_codes, a_sf, a_global, w_codes, w_sf, w_global, bias_bf16,
                           out_bf16, M, N, K, stream, -1, 0);
}

int fp8r_gemm(const uint8_t* a_e4m3, const float* a_row_scale, const uint8_t* w_e4m3,
              const float* w_row_scale, const void* bias_bf16, void* out_bf16, int64_t M,
              int64_t N, int64_t K, bsp_stream_t stream)
{
    return bsp::gemm_entry(false, a_e4m3, nullptr, a_row_scale, w_e4m3, nullptr, w_row_scale,
                           bias_bf16, out_bf16, M, N, K, stream, -1, 0);
}

int bsp_testing_gemm_stall(int scheme, const uint8_t* a, const uint8_t* a_sf, const float* a_scale,
                           const uint8_t* w, const uint8_t* w_sf, const float* w_scale,
                           void* out_bf16, int64_t M, int64_t N, int64_t K,
                           int64_t stop_after_stages, int64_t wait_limit_ms, bsp_stream_t stream)
{
    if (stop_after_stages < 0 || wait_limit_ms <= 0 || wait_limit_ms > 10000)
        return BSP_ERR_INVALID_ARG;
    if (scheme != 0 && scheme != 1) return BSP_ERR_INVALID_ARG;
    return bsp::gemm_entry(scheme == 1, a, a_sf, a_scale, w, w_sf, w_scale, nullptr, out_bf16, M,
                           N, K, stream, stop_after_stages,
                           static_cast<uint64_t>(wait_limit_ms) * 1000000ull);
}

}  // extern "C"
