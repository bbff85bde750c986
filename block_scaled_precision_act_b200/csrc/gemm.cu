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
#include <atomic>
#include <cfloat>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>

#include <cuda.h>
#include <cuda_bf16.h>

#include "bsp_internal.h"
#include "bsp_ptx.cuh"
#include "bsp_testing.h"
#include "nvfp4_block.cuh"

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
    // output re-quantized to NVFP4 instead of written as bf16 (pair kernel, QOUT):
    const float* q_global;           // device fp32 global scale g of the next layer
    uint8_t* q_codes;                // [M][N/2] E2M1 codes of bf16(Y)
    uint8_t* q_sf;                   // E4M3 block scales of bf16(Y), MMA layout, K = N
    // the weight operand (B, its scales) cannot be written by the grid this launch depends
    // on, so the pair producer may fetch the first stages of it before griddep_wait
    // (set only where that grid is the library's own activation quantizer)
    int w_early;
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
    griddep_launch_dependents();   // a dependent grid may start its prologue meanwhile
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
            // Under a programmatic launch the operands may still be being written by
            // the preceding grid (the activation quantizer): nothing is loaded before
            // it has completed.  Everything else in the kernel follows these loads.
            griddep_wait();
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
        int acc_it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            const int mt = tile % num_m, nt = tile / num_m;
            const int a = acc_it % NACC;
            const uint32_t aph = static_cast<uint32_t>((acc_it / NACC) & 1);
            const bool ok = mbar_wait(tfull + a, aph, abort_flag, args.wait_ns, args.status, 4);
            if (!__all_sync(0xffffffffu, ok)) break;   // also reconverges the warp
            tc_fence_after();
            // read here, after the producer's griddep_wait (through the accumulator
            // barrier), so a preceding grid may still be writing the scales at launch
            if constexpr (NVF4) alpha = __fmul_rn(__ldg(args.a_scale), __ldg(args.w_scale));
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

// ---------------------------------------------------------------- CTA-pair kernel
// Two CTAs of a cluster compute one 256 x 256 tile with tcgen05 cta_group::2: CTA r
// loads rows [128r, 128r+128) of the A tile and rows [128r, 128r+128) of the B tile
// (its half of N); the MMA thread of CTA 0 issues one 256x256xK MMA that reads both
// CTAs' shared memory and writes each CTA's 128 x 256 accumulator into that CTA's
// TMEM.  Both CTAs fetch the scale factors of all 256 B rows (no multicast).
//
// Roles (13 warps per CTA):
//   warp 0       TMA producer (both CTAs) into a ring of K-stages of 128 bytes per row;
//   warp 1       TMEM allocation; in CTA 0 one thread issues the MMAs;
//   warps 2..4   (CTA 0, nvfp4) scale-factor copies smem -> TMEM, one chunk kind per
//                warp (A, B rows 0-127, B rows 128-255).  A tcgen05.cp issued by the MMA
//                thread costs it ~48 cycles of issue, serialised with the MMAs; from
//                warps on other sub-partitions the copies overlap the MMAs.  The copies
//                go into a ring of three TMEM scale buffers: with two, the copy warps'
//                handshake (wait for a buffer's release, copy, hand over) does not fit in
//                the one stage of MMAs the ring leaves them, and a K-stage takes ~680
//                cycles instead of ~550 (512 of MMA work).
//   warps 5..12  epilogue, two warps per 32-lane TMEM quadrant, 32-column subtiles.
//                FP8: on a pair's last tile warps 0-3 take two subtiles per quadrant.
// TMEM columns: accumulator 0 = [0, 256), accumulator 1 = [112, 368) (they share 144
// columns), scale buffers at [368, 416), [416, 464) and [464, 512).  The epilogue drains
// the shared columns first and then releases the accumulator, so the next tile's MMAs
// overlap the rest of the epilogue.  Output goes through a 64-byte-swizzled smem slab per
// warp and a TMA store.
template <bool NVF4>
struct PairCfg {
    // A stage holds ATOMS K-atoms (128 rows x 128 bytes each) of A and of B.  NVFP4 keeps
    // one-atom stages so its scale copies pipeline per atom; FP8 takes two-atom stages
    // (half the TMA instructions and barrier round trips per byte).
    static constexpr int ATOMS = NVF4 ? 1 : 2;
    static constexpr int STAGES = NVF4 ? 5 : 3;
    static constexpr int THREADS = 13 * 32;
    static constexpr int ATOM = 128 * kBKB;
    static constexpr int A_BYTES = ATOMS * ATOM;
    static constexpr int B_BYTES = ATOMS * ATOM;
    static constexpr int SFA_BYTES = NVF4 ? 2048 : 0;
    static constexpr int SFB_BYTES = NVF4 ? 4096 : 0;
    static constexpr int K_STAGE = NVF4 ? 256 : 128 * ATOMS;
    static constexpr int K_MMA = NVF4 ? 64 : 32;
    static constexpr int STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int EPI_WARPS = 8;
    static constexpr int EPI_SLAB = 32 * 64;           // one warp's 32 rows x 32 bf16
    static constexpr int OFF_B = STAGES * A_BYTES;
    static constexpr int OFF_SFA = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFB = OFF_SFA + STAGES * SFA_BYTES;
    static constexpr int OFF_EPI = OFF_SFB + STAGES * SFB_BYTES;
    // NVFP4: each epilogue warp's bias columns of the tile (4 subtiles x 32 bf16),
    // fetched while the tile's MMAs run
    static constexpr int BIAS_WARP = NVF4 ? 4 * 32 * 2 : 0;
    static constexpr int OFF_BIAS = OFF_EPI + EPI_WARPS * 2 * EPI_SLAB;
    static constexpr int OFF_BAR = OFF_BIAS + EPI_WARPS * BIAS_WARP;
    static constexpr int SF_NBUF = 3;                  // ring of TMEM scale buffers
    // FP8: warps 0-3 help with the last tile's epilogue (see the kernel's tail)
    static constexpr bool TAIL_HELP = !NVF4;
    static constexpr int NUM_BARS = 2 * STAGES + 2 * SF_NBUF + 5;
    static constexpr int SMEM_BYTES = 1024 + OFF_BAR + NUM_BARS * 8 + 16;
    // accumulator 1 starts at ACC_STRIDE; FP8 keeps no scale buffers, so its accumulators
    // share only 96 columns (3 subtiles), NVFP4's 144 (5 subtiles, the last partly)
    static constexpr int ACC_STRIDE = NVF4 ? 112 : 160;
    static constexpr int SHARED_SUBTILES = (256 - ACC_STRIDE + 31) / 32;
    static constexpr int SF_COL0 = 368;                // three buffers of 48 columns
    static constexpr int SF_BUF = 48;                  // SFA 16 + SFB 32 per K-stage
    static constexpr uint32_t IDESC = NVF4 ? idesc_nvf4(256, 256) : idesc_e4m3(256, 256);
    static_assert(SMEM_BYTES <= 232448, "shared memory budget");
    static_assert(OFF_EPI % 1024 == 0, "epilogue slabs must be 1024-byte aligned");
    static_assert(SF_COL0 + SF_NBUF * SF_BUF <= 512 && (!NVF4 || ACC_STRIDE + 256 <= SF_COL0) &&
                      ACC_STRIDE + 256 <= 512, "TMEM budget");
    static_assert(SHARED_SUBTILES >= 1 && SHARED_SUBTILES <= 6, "shared subtiles");
    static_assert(!NVF4 || ATOMS == 1, "scale copies are staged per atom");
};

template <bool NVF4, bool QOUT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg<NVF4>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmSFA,
                     const __grid_constant__ CUtensorMap tmSFB,
                     const __grid_constant__ CUtensorMap tmY, const GemmArgs args)
{
    static_assert(NVF4 || !QOUT, "the re-quantized output is NVFP4 only");
    griddep_launch_dependents();   // a dependent grid may start its prologue meanwhile
    using C = PairCfg<NVF4>;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* sA = smem;
    uint8_t* sB = smem + C::OFF_B;
    uint8_t* sSFA = smem + C::OFF_SFA;
    uint8_t* sSFB = smem + C::OFF_SFB;
    uint8_t* sEpi = smem + C::OFF_EPI;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + STAGES;
    uint64_t* sf_full = empty + STAGES;     // [SF_NBUF]
    uint64_t* sf_empty = sf_full + C::SF_NBUF;   // [SF_NBUF]
    uint64_t* acc_full = sf_empty + C::SF_NBUF;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* fin = acc_empty + 1;
    uint64_t* cp_fin = fin + 1;             // copy warps' last commits
    uint64_t* help_go = cp_fin + 1;         // the pair's last tile is issued (see the tail)
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(help_go + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int M = args.M, N = args.N, K = args.K;
    const int num_m = (M + 255) / 256;
    const int num_n = (N + 255) / 256;
    const int num_tiles = num_m * num_n;
    const int num_kt = (K + C::K_STAGE - 1) / C::K_STAGE;
    const int kb4 = (K / 16 + 3) / 4;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int b = 0; b < C::SF_NBUF; ++b) {
            mbar_init(sf_full + b, 3);      // one arrive per copy warp
            mbar_init(sf_empty + b, 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 2 * C::EPI_WARPS);   // epilogue warps of both CTAs
        mbar_init(fin, 1);
        mbar_init(cp_fin, 3);
        mbar_init(help_go, 1);
        *abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmY);
        if constexpr (NVF4) {
            prefetch_tmap(&tmSFA);
            prefetch_tmap(&tmSFB);
        }
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_holder, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tbase = *tmem_holder;

    if (warp == 0) {
        // ------------------------------------------------------------ producer (both CTAs)
        if (lane == 0) {
            // A stage's loads: the activation operand (A codes, A scales) and the weight
            // operand (B codes, B scales), all completing on the leader's `full` barrier.
            auto load_a = [&](int st, int kt, int a_row) {
                const uint32_t bar0 = mapa_shared(smem_u32(full + st), 0);
                if constexpr (C::ATOMS == 1) {
                    tma_load_2d_pair(sA + st * C::A_BYTES, &tmA, bar0, kt * kBKB, a_row);
                } else {
                    // operands viewed as [atom][row][128 B]: one box = 128 rows x ATOMS atoms
                    tma_load_3d_pair(sA + st * C::A_BYTES, &tmA, bar0, 0, a_row, C::ATOMS * kt);
                }
                // scale arrays as [row tile][512-byte chunk][64 x 8 bytes]: a stage needs
                // chunks 4kt..4kt+3 of one (A) or two (B) row tiles: one box each
                if constexpr (NVF4)
                    tma_load_3d_pair(sSFA + st * C::SFA_BYTES, &tmSFA, bar0, 0, 4 * kt,
                                     a_row / 128);
            };
            auto load_b = [&](int st, int kt, int b_row, int nt) {
                const uint32_t bar0 = mapa_shared(smem_u32(full + st), 0);
                if constexpr (C::ATOMS == 1)
                    tma_load_2d_pair(sB + st * C::B_BYTES, &tmB, bar0, kt * kBKB, b_row);
                else
                    tma_load_3d_pair(sB + st * C::B_BYTES, &tmB, bar0, 0, b_row, C::ATOMS * kt);
                if constexpr (NVF4)
                    tma_load_3d_pair(sSFB + st * C::SFB_BYTES, &tmSFB, bar0, 0, 4 * kt, nt * 2);
            };
            // The weight operand of the first stages may be fetched before the preceding
            // grid completes (w_early: that grid is the activation quantizer, which does
            // not write it); the ring slots are fresh, so no empty-wait is needed.
            int pre = 0;
            if (args.w_early && pair < num_tiles && args.debug_stop_iter < 0) {
                const int nt0 = pair / num_m;
                pre = num_kt < STAGES ? num_kt : STAGES;
                for (int kt = 0; kt < pre; ++kt) {
                    if (rank == 0) mbar_arrive_expect_tx(full + kt, 2 * C::STAGE_TX);
                    load_b(kt, kt, nt0 * 256 + static_cast<int>(rank) * 128, nt0);
                }
            }
            // Under a programmatic launch the activations may still be being written by
            // the preceding grid (the activation quantizer): none is loaded before it has
            // completed.  Everything else in the kernel follows these loads.
            griddep_wait();
            int64_t it = 0;
            int s = 0;                       // ring slot and its phase, kept incrementally
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
                const int mt = tile % num_m, nt = tile / num_m;
                const int a_row = mt * 256 + static_cast<int>(rank) * 128;
                const int b_row = nt * 256 + static_cast<int>(rank) * 128;
                for (int kt = 0; kt < num_kt; ++kt) {
                    if (it < pre) {              // weight half already issued
                        load_a(s, kt, a_row);
                        ++it;
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1u;
                        }
                        continue;
                    }
                    if (it == args.debug_stop_iter) { ok = false; break; }
                    if (!mbar_wait(empty + s, ph ^ 1u, abort_flag, args.wait_ns, args.status, 11)) {
                        ok = false;
                        break;
                    }
                    // The MMAs release a stage on CTA 0's barrier only; CTA 0 relays it to
                    // CTA 1 with a relaxed arrive (a release-ordered cross-CTA arrive per
                    // stage costs about half the load bandwidth).
                    if (rank == 0 && it >= STAGES)
                        mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(empty + s), 1));
                    if (rank == 0) mbar_arrive_expect_tx(full + s, 2 * C::STAGE_TX);
                    load_a(s, kt, a_row);
                    load_b(s, kt, b_row, nt);
                    ++it;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (rank == 0) {
                for (int64_t i = (it > STAGES ? it - STAGES : 0); i < it; ++i)
                    drain_wait(full + (i % STAGES), static_cast<uint32_t>((i / STAGES) & 1),
                               args.wait_ns, args.status);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (CTA 0)
        if (lane == 0 && rank == 0) {
            int s = 0;                       // ring slot and phase, scale buffer and phase
            uint32_t ph = 0;
            int b = 0;
            uint32_t bph = 0;
            int acc_it = 0;
            bool ok = true;
            // descriptors of ring slot 0; slot s starts s * A_BYTES further on, A_BYTES / 16
            // in the 16-byte address field (no carry: shared memory is below 256 KB)
            const uint64_t adesc0 = sdesc_kmajor_sw128(smem_u32(sA));
            const uint64_t bdesc0 = sdesc_kmajor_sw128(smem_u32(sB));
            for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
                const uint32_t d_tmem = tbase + static_cast<uint32_t>((acc_it & 1) * C::ACC_STRIDE);
                for (int kt = 0; kt < num_kt; ++kt) {
                    // NVFP4: the copy warps hand over a stage's scales only after they have
                    // seen its `full` barrier complete, so waiting on `sf_full` alone also
                    // orders the MMAs after the stage's operand loads (one wait per stage).
                    if (!NVF4 &&
                        !mbar_wait(full + s, ph, abort_flag, args.wait_ns, args.status, 13)) {
                        ok = false;
                        break;
                    }
                    if (NVF4 &&
                        !mbar_wait(sf_full + b, bph, abort_flag, args.wait_ns, args.status, 15)) {
                        ok = false;
                        break;
                    }
                    // A tile's first stage also needs its accumulator back from the epilogue.
                    // Waited for after the stage's operands, which are normally ready long
                    // before: the epilogue's release is the last event of the tile handoff.
                    if (kt == 0 && acc_it > 0 &&
                        !mbar_wait(acc_empty, static_cast<uint32_t>((acc_it - 1) & 1), abort_flag,
                                   args.wait_ns, args.status, 12)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nk = NVF4 ? min(4, K / 64 - 4 * kt)
                                        : min(4 * C::ATOMS,
                                              (K - kt * C::K_STAGE + C::K_MMA - 1) / C::K_MMA);
                    const uint64_t adesc = adesc0 + static_cast<uint64_t>(s * (C::A_BYTES >> 4));
                    const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(s * (C::B_BYTES >> 4));
                    const uint32_t sf = tbase + C::SF_COL0 + b * C::SF_BUF;
                    // K-step k lies in atom k/4 (ATOM bytes further on: ATOM/16 in the
                    // descriptor's address field), 32 bytes (2) per step inside it
                    auto issue = [&](int k) {
                        const uint32_t acc = (kt > 0 || k > 0) ? 1u : 0u;
                        const uint64_t koff = static_cast<uint64_t>((k >> 2) * (C::ATOM >> 4) +
                                                                    2 * (k & 3));
                        if constexpr (NVF4)
                            mma_nvf4_pair(d_tmem, adesc + koff, bdesc + koff, C::IDESC, sf + k * 4,
                                          sf + 16 + k * 8, acc);
                        else
                            mma_f8f6f4_pair(d_tmem, adesc + koff, bdesc + koff, C::IDESC, acc);
                    };
                    // A full K-stage is issued from straight-line code: the same MMAs from a
                    // loop with a run-time trip count cost the issuing thread ~50 cycles
                    // more each, which the tensor pipe cannot hide (measured).  Only a
                    // ragged last stage takes the loop.
                    if (nk == C::K_STAGE / C::K_MMA) {
#pragma unroll
                        for (int k = 0; k < C::K_STAGE / C::K_MMA; ++k) issue(k);
                    } else {
                        for (int k = 0; k < nk; ++k) issue(k);
                    }
                    tc_commit_pair(empty + s, 0x1);
                    if constexpr (NVF4) tc_commit_pair(sf_empty + b, 0x1);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                    if (++b == C::SF_NBUF) {
                        b = 0;
                        bph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit_pair(acc_full, 0x3);
                ++acc_it;
            }
            // every tile of the pair is issued (or the pair gave up): the helpers of the
            // last tile's epilogue may now wait for its accumulator
            if (C::TAIL_HELP && pair < num_tiles) {
                mbar_arrive(help_go);
                mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(help_go), 1));
            }
        }
    } else if (warp <= 4) {
        // ------------------------------------------------------------ scale copies (CTA 0)
        if constexpr (NVF4) {
            if (lane == 0 && rank == 0) {
                const int which = warp - 2;          // 0: SFA, 1: SFB rows 0-127, 2: rows 128-255
                int s = 0;
                uint32_t ph = 0;
                int b = 0;
                uint32_t bph = 0;
                bool ok = true;
                for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
                    for (int kt = 0; kt < num_kt; ++kt) {
                        if (!mbar_wait(sf_empty + b, bph ^ 1u,
                                       abort_flag, args.wait_ns, args.status, 16) ||
                            !mbar_wait(full + s, ph, abort_flag, args.wait_ns, args.status, 17)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const int nk = min(4, K / 64 - 4 * kt);
                        // this warp's chunk kind: destination column and source descriptor of
                        // its first 512-byte chunk; chunk kb is 512 bytes (32 in the
                        // descriptor's 16-byte address field) further on in shared memory
                        // and `dstep` columns further on in TMEM
                        const uint32_t sf = tbase + C::SF_COL0 + b * C::SF_BUF;
                        const uint32_t dst0 = which == 0 ? sf : sf + 16 + (which - 1) * 4;
                        const uint32_t dstep = which == 0 ? 4u : 8u;
                        const uint64_t src0 = sdesc_sf_block(smem_u32(
                            which == 0 ? sSFA + s * C::SFA_BYTES
                                       : sSFB + s * C::SFB_BYTES + (which - 1) * 2048));
                        // straight-line issue for a full stage, as for the MMAs: a run-time
                        // choice or trip count between the copies slows their issue
                        if (nk == 4) {
#pragma unroll
                            for (int kb = 0; kb < 4; ++kb)
                                tmem_cp_32x128b_x4_pair(dst0 + kb * dstep, src0 + 32 * kb);
                        } else {
                            for (int kb = 0; kb < nk; ++kb)
                                tmem_cp_32x128b_x4_pair(dst0 + kb * dstep, src0 + 32 * kb);
                        }
                        // Hand the buffer over with a fence and a plain arrive, not a commit:
                        // the MMAs that read it are issued after this arrive and queue behind
                        // these copies in the pair's in-order tensor pipe, whereas a commit
                        // would complete only after the MMAs already queued ahead of it.
                        tc_fence_before();
                        mbar_arrive(sf_full + b);
                        if (++s == STAGES) {
                            s = 0;
                            ph ^= 1u;
                        }
                        if (++b == C::SF_NBUF) {
                            b = 0;
                            bph ^= 1u;
                        }
                    }
                }
                tc_commit_pair(cp_fin, 0x1);     // lets the teardown wait for every copy
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue (both CTAs)
        const int ew = warp - 5;              // 0..7
        const int q = warp & 3;               // TMEM lane quadrant this warp may access
        const int h = ew >> 2;                // which half of the subtiles
        const uint32_t acc_empty0 = mapa_shared(smem_u32(acc_empty), 0);
        uint8_t* slab0 = sEpi + ew * 2 * C::EPI_SLAB;
        uint8_t* bias_w = smem + C::OFF_BIAS + ew * C::BIAS_WARP;
        // Under a programmatic launch the scales and the bias may still be being written
        // by the preceding grid: these warps read them only after it has completed.
        griddep_wait();
        float alpha = 0.0f;
        float qg = 0.0f, qt = 0.0f;      // re-quantization: g of the next layer and 6g
        if constexpr (NVF4) alpha = __fmul_rn(__ldg(args.a_scale), __ldg(args.w_scale));
        if constexpr (QOUT) {
            qg = __ldg(args.q_global);
            qt = __fmul_rn(6.0f, qg);
        }
        // Subtiles of 32 columns in processing order `ord` (this warp takes the ords of
        // its half h: h, h+2, h+4, h+6).  The ones shared with the other accumulator come
        // first: for NVFP4, columns 112..255 of accumulator 0 are its subtiles 3..7 and
        // columns 0..143 of accumulator 1 its subtiles 0..4 (FP8: 5..7 and 0..2).
        auto subtile_of = [](int ord, int sacc_) {
            return sacc_ == 0 ? (ord + 8 - C::SHARED_SUBTILES) & 7 : ord;
        };
        // NVFP4: this warp's bias columns of a tile, into its smem buffer (lane L: 4
        // columns of subtile L/8); done ahead of the accumulator wait so that the load
        // latency is not on the epilogue's path
        auto fetch_bias = [&](int tile_, int acc_it_) {
            if constexpr (NVF4) {
                if (args.bias == nullptr) return;
                const int ord = 2 * (lane >> 3) + h;
                const int j = subtile_of(ord, acc_it_ & 1);
                const int n = (tile_ / num_m) * 256 + j * 32 + (lane & 7) * 4;
                uint2 v = make_uint2(0u, 0u);
                if (n < N) v = __ldg(reinterpret_cast<const uint2*>(args.bias + n));
                *reinterpret_cast<uint2*>(bias_w + (lane >> 3) * 64 + (lane & 7) * 8) = v;
            }
        };
        const int64_t q_kb4 = N / 64;
        int acc_it = 0;
        int buf = 0;
        int committed = 0;               // bulk-store groups this warp committed
        int last_group[2] = {-1, -1};    // group that last read each slab
        const uint64_t out_policy = l2_policy_evict_first();
        // fp8r: this lane's row scale of the next tile, also fetched ahead
        auto fetch_sa = [&](int tile_) -> float {
            if constexpr (NVF4) {
                return 0.0f;
            } else {
                const int mrow = (tile_ % num_m) * 256 + static_cast<int>(rank) * 128 + q * 32 + lane;
                return mrow < M ? __ldg(args.a_scale + mrow) : 0.0f;
            }
        };
        float sa_next = 0.0f;
        if (pair < num_tiles) {
            fetch_bias(pair, 0);
            sa_next = fetch_sa(pair);
        }
        for (int tile = pair; tile < num_tiles; tile += npairs) {
            const int mt = tile % num_m, nt = tile / num_m;
            __syncwarp();
            const bool ok = mbar_wait(acc_full, static_cast<uint32_t>(acc_it & 1), abort_flag,
                                      args.wait_ns, args.status, 14);
            if (!__all_sync(0xffffffffu, ok)) break;   // also reconverges the warp
            tc_fence_after();
            const int sacc = acc_it & 1;
            const int wrow = mt * 256 + static_cast<int>(rank) * 128 + q * 32;   // warp's first row
            const int m = wrow + lane;
            const float sa = sa_next;
            const uint32_t tq = tbase + (static_cast<uint32_t>(q * 32) << 16) +
                                static_cast<uint32_t>(sacc * C::ACC_STRIDE);
            // The subtiles shared with the other accumulator come first: this warp's share
            // of them (NVFP4: three for half 0, two for half 1; FP8: two and one) is read
            // from TMEM before anything else, then the accumulator is released to the MMA
            // thread.
            uint32_t pre[3][32];
            const int npre = (C::SHARED_SUBTILES + 1 - h) / 2;
#pragma unroll
            for (int idx = 0; idx < 3; ++idx) {
                if (idx < npre) {
                    const int ord = 2 * idx + h;
                    tmem_ld_x32(tq + subtile_of(ord, sacc) * 32, pre[idx]);
                }
            }
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(acc_empty0);   // values are in registers
            // the pair's last tile: orders 6 and 7 go to the tail helpers (below)
            const bool help_tail = C::TAIL_HELP && tile + npairs >= num_tiles;
#pragma unroll
            for (int idx = 0; idx < 4; ++idx) {
                if (idx == 3 && help_tail) continue;
                const int ord = 2 * idx + h;                        // 0..7
                const int j = subtile_of(ord, sacc);
                const int n0 = nt * 256 + j * 32;
                uint32_t r[32];
                if (idx < npre) {
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        r[i] = (idx == 0) ? pre[0][i] : (idx == 1) ? pre[1][i] : pre[2][i];
                } else {
                    tmem_ld_x32(tq + j * 32, r);
                    tmem_ld_wait();
                }
                // a slab this warp may write: the TMA store that last read it must be done
                // reading it
                auto slab_ready = [&]() -> uint8_t* {
                    if (lane == 0 && last_group[buf] >= 0) {
                        if (committed - 1 - last_group[buf] == 0)
                            bulk_wait_group_read<0>();
                        else
                            bulk_wait_group_read<1>();
                    }
                    __syncwarp();
                    return slab0 + buf * C::EPI_SLAB;
                };
                uint32_t packed[16];
                uint8_t* slab = nullptr;
                if (NVF4 && !QOUT && n0 + 32 <= N) {
                    // whole subtile inside N, bf16 out: each 8-column chunk goes to the slab
                    // as soon as it is computed, so that few registers are live beside the
                    // pre-read subtiles
                    slab = slab_ready();
                    const bool has_bias = args.bias != nullptr;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            v[i] = __fmul_rn(__uint_as_float(r[g * 8 + i]), alpha);
                        if (has_bias) {
                            const uint4 bb =
                                *reinterpret_cast<const uint4*>(bias_w + idx * 64 + g * 16);
                            const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                v[2 * i] = __fadd_rn(v[2 * i], bf16lo_to_f32(bw[i]));
                                v[2 * i + 1] = __fadd_rn(v[2 * i + 1], bf16hi_to_f32(bw[i]));
                            }
                        }
                        const int pc = g ^ ((lane >> 1) & 3);           // 64-byte swizzle
                        *reinterpret_cast<uint4*>(slab + lane * 64 + pc * 16) =
                            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                       pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                    }
                } else if (NVF4 && n0 + 32 <= N) {
                    // whole subtile inside N, re-quantized output (which needs all 32 values
                    // in registers): the four bias reads go out before the math
                    uint4 bb[4];
                    const bool has_bias = args.bias != nullptr;
                    if (has_bias) {
#pragma unroll
                        for (int g = 0; g < 4; ++g)
                            bb[g] = *reinterpret_cast<const uint4*>(bias_w + idx * 64 + g * 16);
                    }
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            v[i] = __fmul_rn(__uint_as_float(r[g * 8 + i]), alpha);
                        if (has_bias) {
                            const uint32_t bw[4] = {bb[g].x, bb[g].y, bb[g].z, bb[g].w};
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                v[2 * i] = __fadd_rn(v[2 * i], bf16lo_to_f32(bw[i]));
                                v[2 * i + 1] = __fadd_rn(v[2 * i + 1], bf16hi_to_f32(bw[i]));
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            packed[g * 4 + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int n = n0 + g * 8;
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
                                uint4 bb;
                                if constexpr (NVF4)
                                    bb = *reinterpret_cast<const uint4*>(bias_w + idx * 64 + g * 16);
                                else
                                    bb = __ldg(reinterpret_cast<const uint4*>(args.bias + n));
                                const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    v[2 * i] = __fadd_rn(v[2 * i], bf16lo_to_f32(bw[i]));
                                    v[2 * i + 1] = __fadd_rn(v[2 * i + 1], bf16hi_to_f32(bw[i]));
                                }
                            }
                        }
#pragma unroll
                        for (int i = 0; i < 4; ++i) packed[g * 4 + i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
                    }
                }
                if constexpr (QOUT) {
                    // bf16(Y) re-quantized in registers: this lane's 32 columns are two
                    // whole 16-element blocks of row m (N % 64 == 0)
                    if (m < M && n0 < N) {
                        const uint32_t b0[8] = {packed[0], packed[1], packed[2], packed[3],
                                                packed[4], packed[5], packed[6], packed[7]};
                        const uint32_t b1[8] = {packed[8], packed[9], packed[10], packed[11],
                                                packed[12], packed[13], packed[14], packed[15]};
                        uint32_t sb0, sb1;
                        const uint2 c0 = nvfp4_encode_block16(b0, qg, qt, sb0);
                        const uint2 c1 = nvfp4_encode_block16(b1, qg, qt, sb1);
                        *reinterpret_cast<uint4*>(args.q_codes + static_cast<int64_t>(m) * (N / 2) +
                                                  n0 / 2) = make_uint4(c0.x, c0.y, c1.x, c1.y);
                        *reinterpret_cast<uint16_t*>(args.q_sf +
                                                     sf_mma_offset(m, n0 / 16, q_kb4)) =
                            static_cast<uint16_t>(sb0 | (sb1 << 8));
                    }
                    continue;
                }
                if (slab == nullptr) {
                    slab = slab_ready();
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int pc = c ^ ((lane >> 1) & 3);           // 64-byte swizzle
                        *reinterpret_cast<uint4*>(slab + lane * 64 + pc * 16) =
                            make_uint4(packed[c * 4], packed[c * 4 + 1], packed[c * 4 + 2],
                                       packed[c * 4 + 3]);
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (wrow < M && n0 < N) {
                    if (lane == 0) {
                        tma_store_2d_hint(&tmY, slab, n0, wrow, out_policy);
                        bulk_commit_group();
                    }
                    last_group[buf] = committed++;
                }
                buf ^= 1;
            }
            __syncwarp();                    // every lane has read this tile's bias
            if (tile + npairs < num_tiles) {
                fetch_bias(tile + npairs, acc_it + 1);
                sa_next = fetch_sa(tile + npairs);
            }
            ++acc_it;
        }
        // the stores must have read their smem slabs before the CTA exits
        if (lane == 0) bulk_wait_group_read<0>();
        __syncwarp();
    }

    // ---------------------------------------------------------------- last-tile helpers
    // FP8 (TAIL_HELP): on the pair's last tile the producer and MMA warps and warps 2-3
    // (one per TMEM lane quadrant, idle by then in both CTAs) take the last two subtiles of
    // their quadrant (orders 6 and 7), so each epilogue warp processes three subtiles there
    // instead of four: that epilogue overlaps nothing, and FP8's second warp of a quadrant
    // loads three of its four subtiles after the release (fp8r at 256 x 3072 x 3072:
    // 17.0 -> 15.7 us; the NVFP4 kernel, whose two warps per quadrant are balanced, gained
    // nothing from it).  Their slabs are in the operand ring, which the
    // last tile's completed MMAs no longer read.  They wait on help_go first, which
    // completes once every tile of the pair is issued, so the accumulator phase they then
    // wait for cannot belong to an earlier tile of the same parity.  The arithmetic is the
    // epilogue's generic path (bit-identical outputs).
    if constexpr (C::TAIL_HELP) {
        if (warp < 4 && pair < num_tiles) {
            const int acc_last = (num_tiles - 1 - pair) / npairs;
            const int last_tile = pair + acc_last * npairs;
            // help_go spans the whole GEMM, not one stage or tile, so the per-wait limit
            // (which may be set short) would misfire on long GEMMs; the MMA thread arrives
            // on it even when it gives up, so a 60-second bound is only a safety net
            const uint64_t go_ns = args.wait_ns > 60000000000ull ? args.wait_ns : 60000000000ull;
            __syncwarp();
            const bool hok =
                mbar_wait(help_go, 0, abort_flag, go_ns, args.status, 18) &&
                mbar_wait(acc_full, static_cast<uint32_t>(acc_last & 1), abort_flag,
                          args.wait_ns, args.status, 19);
            if (__all_sync(0xffffffffu, hok)) {
                tc_fence_after();
                // scales and bias may come from the preceding grid
                griddep_wait();
                const int q = warp;
                const int mt = last_tile % num_m, nt = last_tile / num_m;
                const int wrow = mt * 256 + static_cast<int>(rank) * 128 + q * 32;
                const int m = wrow + lane;
                const int sacc = acc_last & 1;
                const uint32_t tq = tbase + (static_cast<uint32_t>(q * 32) << 16) +
                                    static_cast<uint32_t>(sacc * C::ACC_STRIDE);
                const float sa = m < M ? __ldg(args.a_scale + m) : 0.0f;   // row scale
                const uint64_t policy = l2_policy_evict_first();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int ord = 6 + u;
                    const int j = sacc == 0 ? (ord + 8 - C::SHARED_SUBTILES) & 7 : ord;
                    const int n0 = nt * 256 + j * 32;
                    uint32_t r[32];
                    tmem_ld_x32(tq + j * 32, r);
                    tmem_ld_wait();
                    uint8_t* slab = sA + (warp * 2 + u) * C::EPI_SLAB;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int n = n0 + g * 8;
                        float v[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[g * 8 + i]);
                        if (n < N) {
                            const float4 w0 = __ldg(reinterpret_cast<const float4*>(args.w_scale + n));
                            const float4 w1 =
                                __ldg(reinterpret_cast<const float4*>(args.w_scale + n + 4));
                            const float sw[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(__fmul_rn(v[i], sa), sw[i]);
                            if (args.bias != nullptr) {
                                const uint4 bb = __ldg(reinterpret_cast<const uint4*>(args.bias + n));
                                const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    v[2 * i] = __fadd_rn(v[2 * i], bf16lo_to_f32(bw[i]));
                                    v[2 * i + 1] = __fadd_rn(v[2 * i + 1], bf16hi_to_f32(bw[i]));
                                }
                            }
                        }
                        const int pc = g ^ ((lane >> 1) & 3);           // 64-byte swizzle
                        *reinterpret_cast<uint4*>(slab + lane * 64 + pc * 16) =
                            make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                       pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (wrow < M && n0 < N && lane == 0) {
                        tma_store_2d_hint(&tmY, slab, n0, wrow, policy);
                        bulk_commit_group();
                    }
                }
                // the stores must have read their slabs before the CTA exits
                if (lane == 0) bulk_wait_group_read<0>();
                __syncwarp();
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncwarp();
    if (warp == 1 && lane == 0 && rank == 0) {
        tc_commit_pair(fin, 0x1);    // completes once every MMA of the pair is done
        drain_wait(fin, 0, args.wait_ns, args.status);
        if constexpr (NVF4) drain_wait(cp_fin, 0, args.wait_ns, args.status);
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tbase, kTmemCols);
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

// 2-D tensor [rows][inner] of `dtype`, box of box_rows x box_inner elements.
int make_map_2d(CUtensorMap* m, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows,
                CUtensorMapSwizzle swizzle)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return BSP_ERR_CUDA;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {inner * elem_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

// Block scales in the MMA layout as a 3-D tensor of 8-byte elements:
// [row tiles][kb4 chunks of 512 bytes][64]; a box is 4 chunks of `tiles` row tiles.
int make_map_sf(CUtensorMap* m, const void* base, uint64_t kb4, uint64_t row_tiles,
                uint32_t tiles)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return BSP_ERR_CUDA;
    cuuint64_t dims[3] = {64, kb4, row_tiles};
    cuuint64_t strides[2] = {512, kb4 * 512};
    cuuint32_t box[3] = {64, 4, tiles};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

// Operand codes [rows][row_bytes] viewed as [row_bytes/128 atoms][rows][128 B] (the atom
// dimension has the smaller stride); a box is 128 rows x `atoms` atoms, 128-byte swizzle,
// so one TMA instruction brings atoms x 128 bytes of K for 128 rows.  Needs
// row_bytes % 128 == 0.
int make_map_atoms(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
                   uint32_t atoms)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return BSP_ERR_CUDA;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(kBKB), rows, row_bytes / kBKB};
    cuuint64_t strides[2] = {row_bytes, static_cast<cuuint64_t>(kBKB)};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(kBKB), 128, atoms};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? BSP_OK : BSP_ERR_CUDA;
}

// 2-D byte tensor [rows][row_bytes], box of box_rows x 128 bytes, 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows,
             uint32_t box_rows)
{
    return make_map_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, base, row_bytes, rows, kBKB, box_rows,
                       CU_TENSOR_MAP_SWIZZLE_128B);
}

template <bool NVF4, bool QOUT = false>
int launch_pair(const uint8_t* a, const uint8_t* w, const GemmArgs& args, int dev, int sms,
                cudaStream_t s, bool pdl)
{
    using C = PairCfg<NVF4>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t err[kMaxDevices];
    static int max_pairs[kMaxDevices];
    std::call_once(once[dev], [&] {
        err[dev] = cudaFuncSetAttribute(gemm_pair_kernel<NVF4, QOUT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
        if (err[dev] != cudaSuccess) cudaGetLastError();        // no stale error left behind
        max_pairs[dev] = sms / 2;
        if (err[dev] == cudaSuccess) {
            cudaLaunchConfig_t cfg = {};
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 2;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.gridDim = dim3(static_cast<unsigned>(sms), 1, 1);
            cfg.blockDim = dim3(C::THREADS, 1, 1);
            cfg.dynamicSmemBytes = C::SMEM_BYTES;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int clusters = 0;
            if (cudaOccupancyMaxActiveClusters(&clusters, gemm_pair_kernel<NVF4, QOUT>, &cfg) ==
                    cudaSuccess &&
                clusters > 0)
                max_pairs[dev] = clusters < sms / 2 ? clusters : sms / 2;
            else
                cudaGetLastError();
        }
    });
    if (err[dev] != cudaSuccess) return BSP_ERR_CUDA;
    const uint64_t row_bytes = NVF4 ? static_cast<uint64_t>(args.K) / 2 : args.K;
    CUtensorMap tmA, tmB, tmSFA, tmSFB, tmY;
    int st;
    if (C::ATOMS == 1) {
        st = make_map(&tmA, a, row_bytes, static_cast<uint64_t>(args.M), 128);
        if (st == BSP_OK) st = make_map(&tmB, w, row_bytes, static_cast<uint64_t>(args.N), 128);
    } else {
        if (row_bytes % kBKB != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
        st = make_map_atoms(&tmA, a, row_bytes, static_cast<uint64_t>(args.M), C::ATOMS);
        if (st == BSP_OK)
            st = make_map_atoms(&tmB, w, row_bytes, static_cast<uint64_t>(args.N), C::ATOMS);
    }
    if (QOUT)
        std::memset(&tmY, 0, sizeof(tmY));      // no bf16 output: the map is never used
    else if (st == BSP_OK)
        st = make_map_2d(&tmY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, args.out,
                         static_cast<uint64_t>(args.N), static_cast<uint64_t>(args.M), 32, 32,
                         CU_TENSOR_MAP_SWIZZLE_64B);
    if (st != BSP_OK) return st;
    if (NVF4) {
        // scale arrays as [row tile][chunk][64 x 8 bytes]; boxes of 4 chunks x 1 or 2 tiles
        const uint64_t kb4 = static_cast<uint64_t>(args.K / 16 + 3) / 4;
        st = make_map_sf(&tmSFA, args.sfa, kb4, static_cast<uint64_t>(args.M + 127) / 128, 1);
        if (st == BSP_OK)
            st = make_map_sf(&tmSFB, args.sfb, kb4, static_cast<uint64_t>(args.N + 127) / 128, 2);
        if (st != BSP_OK) return st;
    } else {
        tmSFA = tmA;
        tmSFB = tmA;
    }
    const int64_t tiles =
        static_cast<int64_t>((args.M + 255) / 256) * ((args.N + 255) / 256);
    const int pairs = static_cast<int>(tiles < max_pairs[dev] ? tiles : max_pairs[dev]);
    if (launch_kernel(gemm_pair_kernel<NVF4, QOUT>, 2 * pairs, C::THREADS, C::SMEM_BYTES, s, pdl,
                      tmA, tmB, tmSFA, tmSFB, tmY, args) != cudaSuccess) {
        cudaGetLastError();
        return BSP_ERR_CUDA;
    }
    return launch_status();
}

// Kernel choice: 0 = automatic (CTA pairs with 256x256 tiles unless M fits one
// 128-row tile), 1 = CTA pairs, 2 = single CTAs.  Initialised from the
// BSP_GEMM_KERNEL environment variable ("pair" / "single"); tests can set it.
std::atomic<int> g_kernel_choice{-1};

int kernel_choice()
{
    int c = g_kernel_choice.load();
    if (c < 0) {
        const char* e = std::getenv("BSP_GEMM_KERNEL");
        c = (e && std::strcmp(e, "pair") == 0) ? 1 : (e && std::strcmp(e, "single") == 0) ? 2 : 0;
        int expected = -1;
        g_kernel_choice.compare_exchange_strong(expected, c);
        c = g_kernel_choice.load();
    }
    return c;
}

template <bool NVF4, int BN, int STAGES, int NACC>
int launch(const uint8_t* a, const uint8_t* w, const GemmArgs& args, int dev, int sms,
           cudaStream_t s, bool pdl)
{
    using C = Cfg<NVF4, BN, STAGES, NACC>;
    static std::once_flag attr_once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    std::call_once(attr_once[dev], [&] {
        attr_err[dev] = cudaFuncSetAttribute(gemm_kernel<NVF4, BN, STAGES, NACC>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::SMEM_BYTES);
        if (attr_err[dev] != cudaSuccess) cudaGetLastError();   // no stale error left behind
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
    if (launch_kernel(gemm_kernel<NVF4, BN, STAGES, NACC>, grid, kThreads, C::SMEM_BYTES, s, pdl,
                      tmA, tmB, args) != cudaSuccess) {
        cudaGetLastError();
        return BSP_ERR_CUDA;
    }
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

// NVFP4 re-quantization of the output (nvfp4_gemm_quant) instead of a bf16 Y
struct QOut {
    const float* global;
    uint8_t* codes;
    uint8_t* sf;
};

// Every launch allows programmatic stream serialisation: the kernels read no input and
// write no output before their producer's griddep_wait() (the epilogue's reads and
// writes follow it through the pipeline barriers), so a preceding grid that triggers
// early only lets the prologue overlap its tail, and one that does not (any other
// library's kernel) completes first as usual.
int gemm_entry(bool nvf4, const uint8_t* a, const uint8_t* sfa, const float* a_scale,
               const uint8_t* w, const uint8_t* sfb, const float* w_scale, const void* bias,
               void* out, int64_t M, int64_t N, int64_t K, bsp_stream_t stream,
               int64_t debug_stop_iter, uint64_t wait_ns_override, const QOut* q = nullptr,
               bool w_early = false)
{
    const bool pdl = true;
    int st = check_gemm_common(a, w, bias, q ? static_cast<void*>(q->codes) : out, M, N, K);
    if (st != BSP_OK || M == 0 || N == 0) return st;
    if (!a_scale || !w_scale) return BSP_ERR_INVALID_ARG;
    if (q) {
        if (!nvf4 || !q->global || !q->sf) return BSP_ERR_INVALID_ARG;
        if (N % 64 != 0) return BSP_ERR_UNSUPPORTED_SHAPE;
        if (!aligned16(q->sf) || (reinterpret_cast<uintptr_t>(q->global) & 3u))
            return BSP_ERR_MISALIGNED;
    }
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
    args.q_global = q ? q->global : nullptr;
    args.q_codes = q ? q->codes : nullptr;
    args.q_sf = q ? q->sf : nullptr;
    args.w_early = w_early ? 1 : 0;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (q) return launch_pair<true, true>(a, w, args, dev, sms, s, pdl);   // pair kernel only
    const int choice = kernel_choice();
    // the FP8 pair kernel loads whole 128-byte K-atoms (3-D boxes): K % 128 == 0
    const bool pair_ok = nvf4 || K % kBKB == 0;
    const bool pair = pair_ok && (choice == 1 || (choice == 0 && M > kBM));
    if (pair) return nvf4 ? launch_pair<true>(a, w, args, dev, sms, s, pdl)
                          : launch_pair<false>(a, w, args, dev, sms, s, pdl);
    if (nvf4) {
        if (N > 128) return launch<true, 256, 4, 1>(a, w, args, dev, sms, s, pdl);
        return launch<true, 128, 6, 2>(a, w, args, dev, sms, s, pdl);
    }
    if (N > 128) return launch<false, 256, 4, 2>(a, w, args, dev, sms, s, pdl);
    return launch<false, 128, 6, 2>(a, w, args, dev, sms, s, pdl);
}

}  // namespace

int gemm_after_quantizer(bool nvf4, const uint8_t* a, const uint8_t* a_sf, const float* a_scale,
                         const uint8_t* w, const uint8_t* w_sf, const float* w_scale,
                         const void* bias_bf16, void* out_bf16, int64_t M, int64_t N, int64_t K,
                         bsp_stream_t stream)
{
    return gemm_entry(nvf4, a, a_sf, a_scale, w, w_sf, w_scale, bias_bf16, out_bf16, M, N, K,
                      stream, -1, 0, nullptr, true);
}

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

int nvfp4_gemm_quant(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_global,
                     const uint8_t* w_codes, const uint8_t* w_sf, const float* w_global,
                     const void* bias_bf16, const float* out_global, uint8_t* out_codes,
                     uint8_t* out_sf, int64_t M, int64_t N, int64_t K, bsp_stream_t stream)
{
    const bsp::QOut q{out_global, out_codes, out_sf};
    return bsp::gemm_entry(true, a_codes, a_sf, a_global, w_codes, w_sf, w_global, bias_bf16,
                           nullptr, M, N, K, stream, -1, 0, &q);
}

int fp8r_gemm(const uint8_t* a_e4m3, const float* a_row_scale, const uint8_t* w_e4m3,
              const float* w_row_scale, const void* bias_bf16, void* out_bf16, int64_t M,
              int64_t N, int64_t K, bsp_stream_t stream)
{
    return bsp::gemm_entry(false, a_e4m3, nullptr, a_row_scale, w_e4m3, nullptr, w_row_scale,
                           bias_bf16, out_bf16, M, N, K, stream, -1, 0);
}

int bsp_testing_set_gemm_kernel(int choice)
{
    if (choice < 0 || choice > 2) return BSP_ERR_INVALID_ARG;
    const int old = bsp::kernel_choice();
    bsp::g_kernel_choice.store(choice);
    return old;
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
