// Time-batched GEMMs of the LSTM on the sm_100a tensor cores (tcgen05):
// the input projection Gx = X W_ih^T + b over all timesteps ("LSTM Forward
// Computation", Basic Operators: one product with the four gate matrices
// stacked), the weight gradients dW_ih = sum_t da_t x_t^T, dW_hh =
// sum_t da_t h_{t-1}^T (pulsatrix LSTMModule, backward()), and the
// layer-input gradient dX = dG W_ih.
//
// C[M x N] = A[M x K] * B[N x K]^T, each operand K-major in global memory
// (A[m][k] contiguous in k) or MN-major (A stored [K][M], contiguous in m:
// the weight gradient reads dG [B*T][4H] and the layer's sequences
// [B*T][width] as they are).  An MN-major tile lands as BM/32 (bf16: BM/64)
// TMA boxes of [BK K-rows][128 bytes], the layout tcgen05 reads with the
// operand's transpose bit set: bf16 with the 128-byte swizzle, float32 with
// the 128-byte swizzle on 32-byte granules (the one MN-major layout tf32
// operands accept).  A persistent grid (one CTA per SM) walks the BM x BN output tiles
// (bf16 with M >= 1024: 256 x 256, two M = 128 MMAs per K step, so each
// operand byte fetched from L2 feeds twice the products of a 128-row tile);
// warp 0 issues TMA tile loads into a ring of shared-memory stages, warp 1
// (one thread) issues tcgen05.mma into one of two TMEM accumulators, warps
// 4-7 drain the other accumulator through registers to global memory while
// the next tile's MMAs run.  bf16 operands use kind::f16.  float32 operands use three
// kind::tf32 products per K step, hi*hi + hi*lo + lo*hi with hi = x with its
// low 13 mantissa bits cleared and lo = x - hi (exact in fp32).  The stage's
// float32 values are the hi operand as they stand (a tf32 MMA reads the top
// 19 bits of each element); warps 2-3 write the lo tiles beside each stage
// while the hi*hi MMAs of the stage run, and the two cross products follow
// once the lo tiles are in place.  This is the
// error-compensated 3xTF32 scheme of Ootomo & Yokota (2022), "Recovering
// single precision accuracy from Tensor Cores while surpassing the FP32
// theoretical peak performance"; the dropped lo*lo term and the truncation
// of lo keep the product error near 2^-21 relative.
#include <mutex>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"

namespace lstm {
namespace {

// MH: 128-row halves of the tile (one M = 128 MMA each per K step); NACC:
// accumulator sets in tensor memory (2: a tile's epilogue overlaps the next
// tile's MMAs); epilogue warps 4 .. 4 + 4*MH - 1.
template <int KIND> struct Cfg;
template <> struct Cfg<0> {   // bf16, 128 x 256 tiles (small M)
    static constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4, FMT = 1, MH = 1, NACC = 2;
    static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
};
template <> struct Cfg<1> {   // 3xTF32
    static constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3, FMT = 2, MH = 1, NACC = 2;
    static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = 2 * (A_BYTES + B_BYTES);   // hi tiles, then lo tiles
};
template <> struct Cfg<3> {   // 3xTF32, 128 x 256 tiles: half the MMAs per product of Cfg<1>
    static constexpr int BM = 128, BN = 256, BK = 32, STAGES = 2, FMT = 2, MH = 1, NACC = 2;
    static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = 2 * (A_BYTES + B_BYTES);   // hi tiles, then lo tiles
};
template <> struct Cfg<2> {   // bf16, 256 x 256 tiles: a third less operand traffic from L2
    static constexpr int BM = 256, BN = 256, BK = 64, STAGES = 3, FMT = 1, MH = 2, NACC = 1;
    static constexpr int A_BYTES = BM * 128, B_BYTES = BN * 128;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
};

template <int KIND>
constexpr int epi_warps() { return 4 * Cfg<KIND>::MH; }
template <int KIND>
constexpr int threads_of() { return 128 + 32 * epi_warps<KIND>(); }
template <int KIND>
constexpr int stage_floats() { return epi_warps<KIND>() * 32 * 33; }   // one 32 x 33 block per epilogue warp

template <int KIND>
constexpr size_t smem_bytes() {
    return (size_t)Cfg<KIND>::STAGES * Cfg<KIND>::STAGE_BYTES + (size_t)stage_floats<KIND>() * 4 + 1024 + 256;
}

struct TcEpi {
    int M, N, K, k_per_split;
    int tiles_n, tiles_m, splits;   // tile t: n-tile t % tiles_n, then m-tile, then split
    float* C; long long ldc;
    float* C1; long long ldc1; int n_split;
    const float* bias;
    int accumulate;
    int remap_T, remap_B;
    float* ws;                 // split-K partials [splits][M][N] or null
    int* status;
    uint64_t timeout_ns;
    int a_mn, b_mn;            // operand stored MN-major (see launch_tc_gemm)
    int pdl_wait;              // launched as a programmatic dependent: end only after the primary grid
};

__device__ __forceinline__ long long out_row(const TcEpi& e, int m) {
    if (e.remap_T > 0) return (long long)(m % e.remap_T) * e.remap_B + m / e.remap_T;
    if (e.remap_T < 0) return (long long)(m % e.remap_B) * (-e.remap_T) + m / e.remap_B;
    return m;
}

// Drain wait used on the abort path only: ignores the abort flag.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > 100000000ull) break;   // 0.1 s
    }
}

struct TileCoord {
    int m0, n0, split, kbeg, nk;
};

template <int KIND>
__device__ __forceinline__ TileCoord tile_coord(const TcEpi& e, int t) {
    using Cf = Cfg<KIND>;
    TileCoord c;
    const int tn = t % e.tiles_n;
    const int tm = (t / e.tiles_n) % e.tiles_m;
    c.split = t / (e.tiles_n * e.tiles_m);
    c.m0 = tm * Cf::BM;
    c.n0 = tn * Cf::BN;
    c.kbeg = c.split * e.k_per_split;
    const int kend = min(e.K, c.kbeg + e.k_per_split);
    c.nk = kend > c.kbeg ? (kend - c.kbeg + Cf::BK - 1) / Cf::BK : 0;
    return c;
}

// Persistent: block b computes tiles b, b + gridDim.x, ...  Two accumulators
// of BN tensor-memory columns alternate between tiles, so the epilogue of
// one tile overlaps the loads and MMAs of the next.
template <int KIND>
__global__ void __launch_bounds__(threads_of<KIND>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, TcEpi e) {
    using Cf = Cfg<KIND>;
    constexpr int S = Cf::STAGES, BN = Cf::BN, BK = Cf::BK;
    constexpr bool kTf32 = Cf::FMT == 2;   // float32 operands: 3xTF32 with in-place hi/lo split
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    float* stage_out = reinterpret_cast<float*>(smem + S * Cf::STAGE_BYTES);
    uint64_t* full = reinterpret_cast<uint64_t*>(stage_out + stage_floats<KIND>());
    uint64_t* lofull = full + S;
    uint64_t* empty = lofull + S;
    uint64_t* tmem_full = empty + S;       // [2]
    uint64_t* tmem_empty = tmem_full + 2;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tmem_empty + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = e.tiles_n * e.tiles_m * e.splits;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&lofull[s], 64);
            tc::mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            tc::mbar_init(&tmem_full[b], 1);
            tc::mbar_init(&tmem_empty[b], epi_warps<KIND>());   // one arrive per epilogue warp
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, Cf::NACC * Cf::MH * BN);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmA);
            tc::prefetch_tmap(&tmB);
            int it = 0;   // k-chunks issued so far, over all tiles of this block
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const TileCoord c = tile_coord<KIND>(e, t);
                for (int kt = 0; kt < c.nk; ++kt, ++it) {
                    const int s = it % S, r = it / S;
                    if (!tc::mbar_wait(&empty[s], (r & 1) ^ 1, abort_flag, e.status, e.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    unsigned char* st = smem + s * Cf::STAGE_BYTES;
                    tc::mbar_arrive_expect_tx(&full[s], Cf::A_BYTES + Cf::B_BYTES);
                    const int kx = c.kbeg + kt * BK;
                    constexpr int EPB = 128 / (Cf::FMT == 2 ? 4 : 2);   // elements per 128 bytes
                    if (!e.a_mn) {
                        tc::tma_load_2d(st, &tmA, kx, c.m0, &full[s]);
                    } else {
#pragma unroll
                        for (int q = 0; q < Cf::BM / EPB; ++q)
                            tc::tma_load_2d(st + q * BK * 128, &tmA, c.m0 + q * EPB, kx, &full[s]);
                    }
                    if (!e.b_mn) {
                        tc::tma_load_2d(st + Cf::A_BYTES, &tmB, kx, c.n0, &full[s]);
                    } else {
#pragma unroll
                        for (int q = 0; q < BN / EPB; ++q)
                            tc::tma_load_2d(st + Cf::A_BYTES + q * BK * 128, &tmB, c.n0 + q * EPB, kx, &full[s]);
                    }
                }
            }
            if (*abort_flag) {   // let this block's copies land before shared memory is released
                for (int k = it > S ? it - S : 0; k < it; ++k) mbar_drain(&full[k % S], (k / S) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::instr_desc(Cf::FMT, 128, BN) | ((uint32_t)(e.a_mn != 0) << 15) |
                                   ((uint32_t)(e.b_mn != 0) << 16);
            // K step j of an MMA (8 tf32 / 16 bf16 = 32 bytes of a K-major
            // row, or that many 128-byte rows of an MN-major block)
            constexpr uint32_t kMnStep = (Cf::FMT == 2 ? 8 : 16) * 128, kMnLbo = BK * 128;
            const bool amn = e.a_mn != 0, bmn = e.b_mn != 0;
            auto opd = [&](uint32_t base, int j, bool mn) {
                if (!mn) return tc::smem_desc_sw128(base + j * 32);
                return kTf32 ? tc::smem_desc_sw128b32_mn(base + j * kMnStep, kMnLbo)
                             : tc::smem_desc_sw128_mn(base + j * kMnStep, kMnLbo);
            };
            int it = 0, last = -1, i = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++i) {
                const TileCoord c = tile_coord<KIND>(e, t);
                const int ab = i % Cf::NACC;
                // the epilogue has drained this accumulator set (tile i - NACC)
                if (!tc::mbar_wait(&tmem_empty[ab], ((i / Cf::NACC) & 1) ^ 1, abort_flag, e.status, e.timeout_ns))
                    break;
                tc::tc_fence_after();
                const uint32_t acc_t = tmem + (uint32_t)(ab * Cf::MH * BN);
                for (int kt = 0; kt < c.nk; ++kt, ++it) {
                    const int s = it % S, r = it / S;
                    if (!tc::mbar_wait(&full[s], r & 1, abort_flag, e.status, e.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    unsigned char* st = smem + s * Cf::STAGE_BYTES;
                    const uint32_t a_base = tc::smem_u32(st);
                    const uint32_t b_base = a_base + Cf::A_BYTES;
                    if constexpr (!kTf32) {
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint64_t bd = opd(b_base, j, bmn);
                            const uint32_t acc = (kt | j) != 0;
                            // rows [128h, 128h + 128) of the tile: 16 KB further in
                            // either layout (128 K-major rows, or two MN blocks)
#pragma unroll
                            for (int h = 0; h < Cf::MH; ++h)
                                tc::mma_bf16(acc_t + (uint32_t)(h * BN), opd(a_base + h * 16384, j, amn), bd, idesc,
                                             acc);
                        }
                    } else {
                        // hi * hi reads only what the TMA wrote, so it runs
                        // while the split warps write the remainders
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            tc::mma_tf32(acc_t, opd(a_base, j, amn), opd(b_base, j, bmn), idesc, (kt | j) != 0);
                        if (!tc::mbar_wait(&lofull[s], r & 1, abort_flag, e.status, e.timeout_ns)) {
                            tc::mma_commit(&empty[s]);   // the drain below waits for the products issued
                            last = it;
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                        const uint32_t lo_off = Cf::A_BYTES + Cf::B_BYTES;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const uint64_t ad = opd(a_base, j, amn), bd = opd(b_base, j, bmn);
                            tc::mma_tf32(acc_t, opd(a_base + lo_off, j, amn), bd, idesc, 1);   // lo * hi
                            tc::mma_tf32(acc_t, ad, opd(b_base + lo_off, j, bmn), idesc, 1);   // hi * lo
                        }
                    }
                    tc::mma_commit(&empty[s]);
                    last = it;
                }
                if (!ok) break;
                tc::mma_commit(&tmem_full[ab]);
            }
            if (*abort_flag && last >= 0) mbar_drain(&empty[last % S], (last / S) & 1);
        }
    } else if (kTf32 && warp < 4) {
        // hi/lo split of each stage (64 threads), in place for hi.
        const int ct = threadIdx.x - 64;
        int it = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const TileCoord c = tile_coord<KIND>(e, t);
            for (int kt = 0; kt < c.nk; ++kt, ++it) {
                const int s = it % S, r = it / S;
                if (!tc::mbar_wait(&full[s], r & 1, abort_flag, e.status, e.timeout_ns)) {
                    ok = false;
                    break;
                }
                // the stage's float32 values serve as the hi operand as they
                // are (a tf32 MMA reads the top 19 bits of each); only the
                // remainders are written
                const float4* hi = reinterpret_cast<const float4*>(smem + s * Cf::STAGE_BYTES);
                float4* lo = reinterpret_cast<float4*>(smem + s * Cf::STAGE_BYTES + Cf::A_BYTES + Cf::B_BYTES);
                constexpr int NV = (Cf::A_BYTES + Cf::B_BYTES) / 16;
#pragma unroll 4
                for (int i = ct; i < NV; i += 64) {
                    const float4 x = hi[i];
                    float4 l;
                    l.x = x.x - __uint_as_float(__float_as_uint(x.x) & 0xFFFFE000u);
                    l.y = x.y - __uint_as_float(__float_as_uint(x.y) & 0xFFFFE000u);
                    l.z = x.z - __uint_as_float(__float_as_uint(x.z) & 0xFFFFE000u);
                    l.w = x.w - __uint_as_float(__float_as_uint(x.w) & 0xFFFFE000u);
                    lo[i] = l;
                }
                tc::fence_proxy_async_smem();
                tc::mbar_arrive(&lofull[s]);
            }
        }
    } else if (warp >= 4) {
        // Epilogue: each warp drains its 32 accumulator rows in 32 x 32
        // blocks staged through its own shared-memory block, so each global
        // store instruction writes one contiguous 128-byte row segment.
        const int q = warp & 3;               // tensor-memory lane quarter
        const int h = (warp - 4) >> 2;        // 128-row half of the tile
        float* stg = stage_out + (warp - 4) * (32 * 33);
        int i = 0;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
            const TileCoord c = tile_coord<KIND>(e, t);
            const int ab = i % Cf::NACC;
            const bool ok = tc::mbar_wait(&tmem_full[ab], (i / Cf::NACC) & 1, abort_flag, e.status, e.timeout_ns);
            if (!ok) break;
            tc::tc_fence_after();
            const uint32_t acc_t =
                tmem + (uint32_t)(ab * Cf::MH * BN + h * BN) + ((uint32_t)(q * 32) << 16);
            // Output row of accumulator row (q*32 + lane), computed once per
            // tile and broadcast inside the row loop.
            const int rbase = c.m0 + h * 128 + q * 32;
            const int mrow = rbase + lane;
            const long long my_row = e.ws ? (long long)mrow : out_row(e, mrow);
            const int rows_here = min(32, e.M - rbase);
            for (int cc = 0; cc < BN; cc += 32) {
                float v[16], w[16];
                tc::tmem_ld16(acc_t + (uint32_t)cc, v);
                tc::tmem_ld16(acc_t + (uint32_t)(cc + 16), w);
                tc::tmem_ld_wait();
                if (cc + 32 >= BN) {
                    // every column of this accumulator is in registers: hand
                    // it back to the MMA warp before the stores
                    tc::tc_fence_before();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(&tmem_empty[ab]);
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    stg[lane * 33 + k] = c.nk ? v[k] : 0.f;
                    stg[lane * 33 + 16 + k] = c.nk ? w[k] : 0.f;
                }
                __syncwarp();
                const int n = c.n0 + cc + lane;
                const bool ncol = n < e.N;
                const float bn = (!e.ws && e.bias && ncol) ? e.bias[n] : 0.f;
                float* base;
                long long ld;
                if (e.ws) {
                    base = e.ws + (size_t)c.split * e.M * e.N + n;
                    ld = e.N;
                } else if (n < e.n_split) {
                    base = e.C + n;
                    ld = e.ldc;
                } else {
                    base = e.C1 + (n - e.n_split);
                    ld = e.ldc1;
                }
#pragma unroll 8
                for (int rr = 0; rr < 32; ++rr) {
                    const long long row = __shfl_sync(0xffffffffu, my_row, rr);
                    if (rr < rows_here && ncol) {
                        float* dst = base + row * ld;
                        float val = stg[rr * 33 + lane] + bn;
                        if (e.accumulate) val += *dst;
                        *dst = val;
                    }
                }
                __syncwarp();
            }
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, Cf::NACC * Cf::MH * BN);
    }
    // A programmatic dependent of a recurrence ran beside it; it completes only
    // after that grid has, so work behind it in the stream stays ordered after both.
    if (e.pdl_wait) asm volatile("griddepcontrol.wait;" ::: "memory");
}

__global__ void splitk_reduce_kernel(TcEpi e, int splits) {
    const long long total = (long long)e.M * e.N;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int m = (int)(i / e.N), n = (int)(i % e.N);
        float val = 0.f;
        for (int z = 0; z < splits; ++z) val += e.ws[(size_t)z * total + i];
        val += e.bias ? e.bias[n] : 0.f;
        const long long row = out_row(e, m);
        float* dst = n < e.n_split ? e.C + row * e.ldc + n : e.C1 + row * e.ldc1 + (n - e.n_split);
        if (e.accumulate) val += *dst;
        *dst = val;
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// mn32: a float32 MN-major operand (128-byte swizzle on 32-byte granules)
bool make_map(CUtensorMap* map, DType dt, const void* base, long long rows, long long cols, long long ld,
              int box_rows, bool mn32 = false) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    const size_t es = dtype_size(dt);
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ld * es)};
    cuuint32_t box[2] = {(cuuint32_t)(128 / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, dt == DType::F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     mn32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int KIND>
cudaError_t launch_kind(const TcGemmArgs& g, cudaStream_t s, int* nlaunch) {
    using Cf = Cfg<KIND>;
    CUtensorMap ta, tb;
    // K-major: [M][K] rows, boxes of BM rows; MN-major: [K][M] rows, boxes of
    // BK rows (128 bytes of M each)
    const bool f32 = g.dt == DType::F32;
    if (!(g.a_mn ? make_map(&ta, g.dt, g.A, g.K, g.M, g.lda, Cf::BK, f32)
                 : make_map(&ta, g.dt, g.A, g.M, g.K, g.lda, Cf::BM)))
        return cudaErrorInvalidValue;
    if (!(g.b_mn ? make_map(&tb, g.dt, g.B, g.K, g.N, g.ldb, Cf::BK, f32)
                 : make_map(&tb, g.dt, g.B, g.N, g.K, g.ldb, Cf::BN)))
        return cudaErrorInvalidValue;
    TcEpi e{};
    e.a_mn = g.a_mn; e.b_mn = g.b_mn;
    e.M = g.M; e.N = g.N; e.K = g.K;
    const int kchunks = (g.K + Cf::BK - 1) / Cf::BK;
    const int sms = g.num_sms > 0 ? g.num_sms : 148;
    const long long tiles = (long long)((g.N + Cf::BN - 1) / Cf::BN) * ((g.M + Cf::BM - 1) / Cf::BM);
    // Split K when the tiles fill the SMs poorly and partial sums fit in
    // g.ws: the split count (<= g.splitk) with the best last-wave occupancy,
    // each split keeping at least 16 K chunks.
    int splits = 1;
    if (g.ws && g.splitk > 1) {
        auto occ = [&](long long u) { return (double)u / (double)(((u + sms - 1) / sms) * sms); };
        double best = occ(tiles);
        for (int sp = 2; sp <= g.splitk; ++sp) {
            if (kchunks / sp < 16 || (long long)sp * g.M * g.N > g.ws_floats) break;
            if (occ(tiles * sp) > best + 0.05) {
                best = occ(tiles * sp);
                splits = sp;
            }
        }
    }
    e.k_per_split = ((kchunks + splits - 1) / splits) * Cf::BK;
    e.C = g.C; e.ldc = g.ldc;
    e.C1 = g.C1 ? g.C1 : g.C; e.ldc1 = g.C1 ? g.ldc1 : g.ldc;
    e.n_split = g.C1 ? g.n_split : g.N;
    e.bias = g.bias; e.accumulate = g.accumulate;
    e.remap_T = g.remap_T; e.remap_B = g.remap_B;
    e.ws = splits > 1 ? g.ws : nullptr;
    e.status = g.status; e.timeout_ns = g.timeout_ns;
    const size_t smem = smem_bytes<KIND>();
    cudaError_t err = cudaFuncSetAttribute(tc_gemm_kernel<KIND>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)smem);
    if (err != cudaSuccess) return err;
    e.tiles_n = (g.N + Cf::BN - 1) / Cf::BN;
    e.tiles_m = (g.M + Cf::BM - 1) / Cf::BM;
    e.splits = splits;
    const long long ntiles = (long long)e.tiles_n * e.tiles_m * splits;
    const int grid = (int)std::min<long long>(ntiles, sms);
    if (g.pdl) {
        // starts once every block of the preceding kernel in the stream (a
        // persistent recurrence) has signalled; runs on the SMs it leaves free
        e.pdl_wait = 1;
        cudaLaunchConfig_t cfg{};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(threads_of<KIND>());
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        err = cudaLaunchKernelEx(&cfg, tc_gemm_kernel<KIND>, ta, tb, e);
    } else {
        tc_gemm_kernel<KIND><<<grid, threads_of<KIND>(), smem, s>>>(ta, tb, e);
        err = cudaGetLastError();
    }
    if (nlaunch) *nlaunch = 1;
    if (err != cudaSuccess || splits == 1) return err;
    const long long total = (long long)g.M * g.N;
    const int blocks = (int)std::min<long long>((total + 255) / 256, 148LL * 8);
    splitk_reduce_kernel<<<blocks, 256, 0, s>>>(e, splits);
    if (nlaunch) *nlaunch = 2;
    return cudaGetLastError();
}

}  // namespace

bool tc_gemm_supported(const TcGemmArgs& g) {
    if (g.M <= 0 || g.N <= 0 || g.K <= 0) return false;
    if (!encode_fn()) return false;
    const size_t es = dtype_size(g.dt);
    if ((g.lda * es) % 16 != 0 || (g.ldb * es) % 16 != 0) return false;
    if ((reinterpret_cast<uintptr_t>(g.A) & 15) || (reinterpret_cast<uintptr_t>(g.B) & 15)) return false;
    // the contiguous dimension of each operand spans at least one 128-byte box
    const long long inner = 128 / (long long)es;
    if ((g.a_mn ? g.M : g.K) < inner || (g.b_mn ? g.N : g.K) < inner) return false;
    return true;
}

cudaError_t launch_tc_gemm(const TcGemmArgs& g, cudaStream_t s, int* nlaunch) {
    if (g.dt == DType::F32) {
        // 128 x 256 tiles halve the MMAs per product but halve the tile count:
        // used when they still fill the SMs or K can be split
        const long long tiles3 = (long long)((g.M + Cfg<3>::BM - 1) / Cfg<3>::BM) * ((g.N + Cfg<3>::BN - 1) / Cfg<3>::BN);
        const int sms = g.num_sms > 0 ? g.num_sms : 148;
        const bool wide = g.N >= Cfg<3>::BN && (tiles3 >= sms || (g.ws && g.splitk > 1));
        return wide ? launch_kind<3>(g, s, nlaunch) : launch_kind<1>(g, s, nlaunch);
    }
    return g.M >= 4 * Cfg<2>::BM ? launch_kind<2>(g, s, nlaunch) : launch_kind<0>(g, s, nlaunch);
}

// ---------------------------------------------------------------- transposes
namespace {

template <bool BF>
__device__ __forceinline__ float ld_elem(const void* p, long long i) {
    if constexpr (BF) return __bfloat162float(static_cast<const bf16*>(p)[i]);
    return static_cast<const float*>(p)[i];
}

template <bool BF>
__device__ __forceinline__ void st_elem(void* p, long long i, float v) {
    if constexpr (BF)
        static_cast<bf16*>(p)[i] = __float2bfloat16_rn(v);
    else
        static_cast<float*>(p)[i] = v;
}

// Tiles of 32 rows (m) x 64 columns (c), 32 x 8 threads: each thread's eight
// source elements are all loaded (predicated) before any goes to shared
// memory, so their latencies overlap.
constexpr int kTrM = 32, kTrC = 64;
template <int MODE, bool SB, bool DB>
__global__ void __launch_bounds__(256) transpose_kernel(TransposeArgs a) {
    __shared__ float tile[kTrM][kTrC + 1];
    const int m0 = blockIdx.x * kTrM, c0 = blockIdx.y * kTrC;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
    float v[4][2];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
        const int m = m0 + ty + 8 * r;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int c = c0 + 32 * h + tx;
            v[r][h] = 0.f;
            if (m < a.M && c < a.C) {
                if (MODE == 0) {
                    long long row = m;
                    if (a.bt_remap) row = (long long)(m % a.B) * a.T + m / a.B;   // m = t*B + b -> b*T + t
                    v[r][h] = ld_elem<SB>(a.src, row * a.lds + c);
                } else {   // h_{t-1} in the direction's order, h0 at its first step
                    const int t = m / a.B, b = m % a.B;
                    const int ts = a.dir == 0 ? t - 1 : t + 1;
                    if (ts >= 0 && ts < a.T)
                        v[r][h] = ld_elem<SB>(a.src, ((long long)ts * a.B + b) * a.lds + c);
                    else if (a.h0)
                        v[r][h] = ld_elem<SB>(a.h0, (long long)b * a.C + c);
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int h = 0; h < 2; ++h) tile[ty + 8 * r][32 * h + tx] = v[r][h];
    __syncthreads();
    const int m = m0 + tx;
#pragma unroll
    for (int r = 0; r < kTrC / 8; ++r) {
        const int cl = ty + 8 * r, cc = c0 + cl;
        if (m < a.M && cc < a.C) st_elem<DB>(a.dst, (long long)cc * a.ldd + m, tile[tx][cl]);
    }
}

template <int MODE>
cudaError_t launch_transpose_mode(const TransposeArgs& a, dim3 grid, cudaStream_t s) {
    if (a.src_bf16) {
        if (a.dst_bf16) transpose_kernel<MODE, true, true><<<grid, 256, 0, s>>>(a);
        else transpose_kernel<MODE, true, false><<<grid, 256, 0, s>>>(a);
    } else {
        if (a.dst_bf16) transpose_kernel<MODE, false, true><<<grid, 256, 0, s>>>(a);
        else transpose_kernel<MODE, false, false><<<grid, 256, 0, s>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_transpose(const TransposeArgs& a, cudaStream_t s) {
    if (a.M <= 0 || a.C <= 0) return cudaSuccess;
    dim3 grid((a.M + kTrM - 1) / kTrM, (a.C + kTrC - 1) / kTrC);
    return a.mode == 0 ? launch_transpose_mode<0>(a, grid, s) : launch_transpose_mode<1>(a, grid, s);
}

}  // namespace lstm
