// Persistent LSTM forward recurrence on the sm_100a tensor cores (bf16).
//
// Each step computes, for every direction d, the gate pre-activations
//     a[p][b] = sum_k W_hh[p][k] h_{t-1}[b][k] + Gx[t][b][p]
// (warp_nn "Long Short-Term Memory (LSTM)" equation block; Gx holds
// W_ih x_t + b_ih + b_hh from the time-batched projection) and the cell
// update c = f c + i g, h = o tanh(c).
//
// Block (d, bg, j) owns 128 packed gate rows p = 4u + q of units
// [32j, 32j+32) and the batch rows of group bg, and keeps its whole W_hh
// slice resident for the sequence: K chunks [0, kc_smem) in shared memory
// (128-byte-swizzled K-major tiles loaded once by TMA) and the remaining
// chunks in tensor memory, where tcgen05.mma reads them as the A operand.
// The accumulator (128 lanes x N batch columns, fp32) also lives in tensor
// memory.  One step:
//   warp 0:         wait for the group's h_{t-1}, TMA it (N rows x 64 k per
//                   chunk) through a ring of shared-memory stages
//   warp 1:         once the accumulator holds Gx[t] (d_ready), one thread
//                   issues M=128 x N x K=16 MMAs over all of K
//   epilogue warps: (two per tensor-memory lane quarter, each half of the
//                   batch columns) tcgen05.ld the pre-activations, exchange
//                   the four gates of each unit inside 4-lane groups
//                   (shuffles), update c (registers) and h, write h_t and
//                   arrive on the counter; then load Gx[t+1] and store it
//                   into the accumulator (tcgen05.st) and signal d_ready.
// Only bf16 inference uses this kernel; every wait is bounded.
#include <algorithm>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"

namespace lstm {
namespace {

constexpr int kRows = 128;             // gate rows per block
constexpr int kChunkW = kRows * 128;   // bytes of one 64-wide K chunk of W
constexpr int kMaxNcc = 8;             // N <= 128 batch columns per block
constexpr int kNccHalf = kMaxNcc / 2;  // 16-column chunks per epilogue half
constexpr int kEpi = 256;              // epilogue threads: warps 2-9, two per lane quarter
constexpr int kThreads = 64 + kEpi;    // warp 0 TMA, warp 1 MMA
constexpr uint32_t kAcol = 256;        // tensor-memory column of the resident W part

struct TcRecParams {
    int H, B, T, D;
    int nbg, Bg, N, nu, kc_smem, stages;
    const float* gx;          // [T][B][D*G] packed rows, biases included
    const float* c0;          // [D][B][H] or null
    bf16* hx;                 // [D][T+1][B][H]; slot 0 holds h0
    bf16* hseq;               // [T][B][D*H] or null
    bf16* out; long long out_st, out_sb;
    bf16* h_n; float* c_n;    // [D][B][H]
    const bf16* wpk;          // [D*G][H] packed rows
    unsigned* ctr;            // [D*nbg]
    int* status;
    uint64_t timeout_ns;
};

// Branch-free choice among four registers by a lane-dependent index k in
// [0, 4): two levels of selp, so a warp never diverges on it.
__device__ __forceinline__ float selp_f(float a, float b, uint32_t take_b) {
    float r;
    asm("{\n\t.reg .pred p;\n\tsetp.ne.u32 p, %3, 0;\n\tselp.f32 %0, %2, %1, p;\n\t}"
        : "=f"(r) : "f"(a), "f"(b), "r"(take_b));
    return r;
}

__device__ __forceinline__ float sel4(float a0, float a1, float a2, float a3, int k) {
    const float lo = selp_f(a0, a1, (uint32_t)k & 1u);
    const float hi = selp_f(a2, a3, (uint32_t)k & 1u);
    return selp_f(lo, hi, (uint32_t)k & 2u);
}

// Gate nonlinearities of this bf16-only kernel: CUDA's fast intrinsics and the
// hardware tanh approximation (relative error near 2^-11, far inside the bf16
// path's 2e-2 tolerance).
__device__ __forceinline__ float sigmoid_fast(float z) { return __fdividef(1.f, 1.f + __expf(-z)); }

__device__ __forceinline__ float tanh_fast(float z) {
    float r;
    asm("tanh.approx.f32 %0, %1;" : "=f"(r) : "f"(z));
    return r;
}

__device__ __forceinline__ bool named_bar_or(int id, int n, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Bounded wait until *ctr >= target (single thread).
__device__ __forceinline__ bool ctr_wait(const unsigned* ctr, unsigned target, volatile int* abort, int* status,
                                         uint64_t timeout_ns) {
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    unsigned it = 0;
    while (ld_acquire(ctr) < target) {
        if ((++it & 63u) == 0) {
            if (*abort || ld_volatile(status) != kStatusOk) {
                *abort = 1;
                return false;
            }
            if (globaltimer_ns() - t0 > timeout_ns) {
                atomicCAS(status, kStatusOk, kStatusTimeout);
                *abort = 1;
                return false;
            }
        }
    }
    return true;
}

// Gx[t] of accumulator row `prow - prow0` (packed row prow) for columns
// [cbase, cbase + NH) of this thread's half, written into the accumulator
// (zeros outside the batch), then d_ready.  Two groups of 32 columns: each
// group's loads are all in flight before its tensor-memory stores.
__device__ __forceinline__ void preload_gx(const float* gx, int t, int B, size_t ldgx, int prow, int b0,
                                           int cbase, int NH, int nB, uint32_t trow, uint64_t* d_ready) {
    const float* gxp = gx + (size_t)t * B * ldgx + (size_t)prow;
#pragma unroll
    for (int g = 0; g < kNccHalf / 2; ++g) {
        if (32 * g >= NH) break;
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int col = cbase + 32 * g + i;
            v[i] = (32 * g + i < NH && col < nB) ? __float_as_uint(__ldg(gxp + (size_t)(b0 + col) * ldgx)) : 0u;
        }
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) { lo[i] = v[i]; hi[i] = v[16 + i]; }
        tc::tmem_st16(trow + (uint32_t)(cbase + 32 * g), lo);
        if (32 * g + 16 < NH) tc::tmem_st16(trow + (uint32_t)(cbase + 32 * g + 16), hi);
    }
    tc::tmem_st_wait();
    tc::tc_fence_before();
    tc::mbar_arrive(d_ready);
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > 100000000ull) break;
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_rec_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW, TcRecParams a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int KT = H / 64, S = a.stages, N = a.N;
    const int hstage = N * 128;
    unsigned char* sW = smem;
    unsigned char* sH = smem + a.kc_smem * kChunkW;
    uint64_t* full = reinterpret_cast<uint64_t*>(sH + S * hstage);
    uint64_t* empty = full + S;
    uint64_t* d_ready = empty + S;
    uint64_t* mma_done = d_ready + 1;
    uint64_t* w_full = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(w_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int j = blockIdx.x % a.nu;
    const int bg = (blockIdx.x / a.nu) % a.nbg;
    const int d = blockIdx.x / (a.nu * a.nbg);
    const int b0 = bg * a.Bg, nB = min(a.Bg, B - b0);
    const int prow0 = d * G + j * kRows;
    unsigned* ctr = a.ctr + d * a.nbg + bg;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(d_ready, kEpi);
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(w_full, 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Resident weights: shared-memory part by TMA, tensor-memory part by the
    // epilogue warps (row r of the block on lane r; two bf16 per column).
    if (warp == 0 && lane == 0) {
        tc::prefetch_tmap(&tmH);
        tc::prefetch_tmap(&tmW);
        if (a.kc_smem > 0) {
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(a.kc_smem * kChunkW));
            for (int c = 0; c < a.kc_smem; ++c) tc::tma_load_2d(sW + c * kChunkW, &tmW, 64 * c, prow0, w_full);
        }
    }
    const int q = warp & 3;                 // lane quarter of an epilogue warp
    const int r = q * 32 + lane;            // accumulator row of this epilogue thread
    const int half = (warp - 2) >> 2;       // batch-column half of an epilogue warp
    if (warp >= 2 && half == 0) {
        const bf16* wrow = a.wpk + (size_t)(prow0 + r) * H;
        for (int c = a.kc_smem; c < KT; ++c) {
            const uint4* src = reinterpret_cast<const uint4*>(wrow + 64 * c);
            uint32_t v0[16], v1[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 x = src[i];
                v0[4 * i] = x.x; v0[4 * i + 1] = x.y; v0[4 * i + 2] = x.z; v0[4 * i + 3] = x.w;
                const uint4 y = src[4 + i];
                v1[4 * i] = y.x; v1[4 * i + 1] = y.y; v1[4 * i + 2] = y.z; v1[4 * i + 3] = y.w;
            }
            const uint32_t col = kAcol + (uint32_t)(c - a.kc_smem) * 32;
            tc::tmem_st16(tmem + ((uint32_t)(q * 32) << 16) + col, v0);
            tc::tmem_st16(tmem + ((uint32_t)(q * 32) << 16) + col + 16, v1);
        }
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    if (warp == 0) {
        // ------------------------------------------------------ h producer
        if (lane == 0) {
            int issued = 0;
            bool ok = true;
            for (int s = 0; s < T && ok; ++s) {
                if (s > 0) {
                    if (!ctr_wait(ctr, (unsigned)(a.nu * s), abort_flag, a.status, a.timeout_ns)) break;
                    tc::fence_proxy_async_global();
                }
                const int row0 = (d * (T + 1) + s) * B + b0;
                for (int c = 0; c < KT; ++c) {
                    const int idx = s * KT + c, st = idx % S, rnd = idx / S;
                    if (!tc::mbar_wait(&empty[st], (rnd & 1) ^ 1, abort_flag, a.status, a.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[st], (uint32_t)hstage);
                    tc::tma_load_2d(sH + st * hstage, &tmH, 64 * c, row0, &full[st]);
                    issued = idx + 1;
                }
            }
            if (*abort_flag) {
                for (int idx = issued > S ? issued - S : 0; idx < issued; ++idx)
                    drain_wait(&full[idx % S], (idx / S) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc = tc::instr_desc(1, kRows, N);
            bool ok = a.kc_smem == 0 || tc::mbar_wait(w_full, 0, abort_flag, a.status, a.timeout_ns);
            int last = -1;
            for (int s = 0; s < T && ok; ++s) {
                if (!tc::mbar_wait(d_ready, s & 1, abort_flag, a.status, a.timeout_ns)) break;
                tc::tc_fence_after();
                for (int c = 0; c < KT; ++c) {
                    const int idx = s * KT + c, st = idx % S, rnd = idx / S;
                    if (!tc::mbar_wait(&full[st], rnd & 1, abort_flag, a.status, a.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t b_base = tc::smem_u32(sH + st * hstage);
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        const uint64_t bd = tc::smem_desc_sw128(b_base + 32 * jj);
                        if (c < a.kc_smem) {
                            const uint64_t ad = tc::smem_desc_sw128(tc::smem_u32(sW + c * kChunkW) + 32 * jj);
                            tc::mma_bf16(tmem, ad, bd, idesc, 1);
                        } else {
                            const uint32_t at = tmem + kAcol + (uint32_t)(c - a.kc_smem) * 32 + 8 * jj;
                            tc::mma_bf16_ts(tmem, at, bd, idesc, 1);
                        }
                    }
                    tc::mma_commit(&empty[st]);
                    last = idx;
                }
                if (!ok) break;
                tc::mma_commit(mma_done);
            }
            if (*abort_flag && last >= 0) drain_wait(&empty[last % S], (last / S) & 1);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int gq = lane & 3;                    // gate of this lane's row
        const int u = j * 32 + q * 8 + (lane >> 2); // unit of this lane's row group
        const int NH = N / 2;                       // columns of this half (multiple of 16)
        const int cbase = half * NH;                // first column of this half
        float creg[kNccHalf][4];
#pragma unroll
        for (int cc = 0; cc < kNccHalf; ++cc)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int col = cbase + 16 * cc + 4 * gq + i;
                creg[cc][i] = (16 * cc < NH && col < nB && a.c0) ? a.c0[((size_t)d * B + b0 + col) * H + u] : 0.f;
            }
        const size_t ldgx = (size_t)D * G;
        const size_t ldseq = (size_t)D * H;
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        preload_gx(a.gx, d == 0 ? 0 : T - 1, B, ldgx, prow0 + r, b0, cbase, NH, nB, trow, d_ready);
        for (int s = 0; s < T; ++s) {
            const int t = d == 0 ? s : T - 1 - s;
            const bool ok = tc::mbar_wait(mma_done, s & 1, abort_flag, a.status, a.timeout_ns);
            if (named_bar_or(1, kEpi, !ok)) break;   // every epilogue thread leaves together
            tc::tc_fence_after();
            bf16* hxo = a.hx + ((size_t)(d * (T + 1) + s + 1) * B) * H;
#pragma unroll
            for (int cc = 0; cc < kNccHalf; ++cc) {
                if (16 * cc >= NH) break;
                float v[16];
                tc::tmem_ld16(trow + (uint32_t)(cbase + 16 * cc), v);
                tc::tmem_ld_wait();
                // v[4k + i]: gate gq at column 16cc + 4k + i.  Three xor
                // exchanges inside each 4-lane group give lane gq all four
                // gates at column 16cc + 4gq + i (gate X arrives in round gq ^ X).
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float rcv[4];
                    rcv[0] = sel4(v[i], v[4 + i], v[8 + i], v[12 + i], gq);
#pragma unroll
                    for (int rr = 1; rr < 4; ++rr)
                        rcv[rr] = __shfl_xor_sync(0xffffffffu, sel4(v[i], v[4 + i], v[8 + i], v[12 + i], gq ^ rr), rr);
                    const float pi = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 0);
                    const float pf = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 1);
                    const float pgg = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 2);
                    const float po = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 3);
                    const int col = cbase + 16 * cc + 4 * gq + i;
                    if (col >= nB) continue;
                    const int b = b0 + col;
                    const float ig = sigmoid_fast(pi), fg = sigmoid_fast(pf), gg = tanh_fast(pgg);
                    const float og = sigmoid_fast(po);
                    const float c = fg * creg[cc][i] + ig * gg;
                    creg[cc][i] = c;
                    const bf16 hv = __float2bfloat16_rn(og * tanh_fast(c));
                    hxo[(size_t)b * H + u] = hv;
                    if (a.hseq) a.hseq[((size_t)t * B + b) * ldseq + (size_t)d * H + u] = hv;
                    if (a.out) a.out[(size_t)t * a.out_st + (size_t)b * a.out_sb + (size_t)d * H + u] = hv;
                    if (s == T - 1) {
                        a.h_n[((size_t)d * B + b) * H + u] = hv;
                        a.c_n[((size_t)d * B + b) * H + u] = c;
                    }
                }
            }
            // publish h_t to the group, then hand the accumulator Gx[t+1]
            tc::fence_proxy_async_global();
            tc::named_bar_sync(1, kEpi);
            if (warp == 2 && lane == 0) {
                __threadfence();
                atomicAdd(ctr, 1u);
            }
            // Gx[t+1]: its load latency overlaps the group barrier and the h
            // TMA that the next step's MMAs wait for anyway
            if (s + 1 < T)
                preload_gx(a.gx, d == 0 ? s + 1 : T - 2 - s, B, ldgx, prow0 + r, b0, cbase, NH, nB, trow, d_ready);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
}

}  // namespace

TcRecPlan plan_tc_rec(int H, int B, int D, int num_sms, size_t smem_max) {
    TcRecPlan p{};
    if (H % 64 != 0 || B < 1) return p;
    const int KT = H / 64;
    const int nu = 4 * H / kRows;
    const int kc_smem = std::max(0, KT - 8);
    const int max_groups = num_sms / (D * nu);
    if (max_groups < 1) return p;
    int nbg = std::min(max_groups, std::max(1, (B + 31) / 32));
    int Bg = (B + nbg - 1) / nbg;
    while (((Bg + 31) / 32) * 32 > 16 * kMaxNcc && nbg < max_groups) {
        ++nbg;
        Bg = (B + nbg - 1) / nbg;
    }
    const int N = ((Bg + 31) / 32) * 32;   // two halves of whole 16-column chunks
    if (N > 16 * kMaxNcc) return p;
    if (nbg > 1 && (nbg - 1) * Bg >= B) return p;
    const size_t fixed = (size_t)kc_smem * kChunkW + 1024 + 256;
    int stages = 8;
    while (stages >= 2 && fixed + (size_t)stages * N * 128 > smem_max) --stages;
    if (stages < 2) return p;
    p.ok = true;
    p.nbg = nbg; p.Bg = Bg; p.N = N; p.nu = nu; p.kc_smem = kc_smem; p.stages = stages;
    p.ctas = D * nbg * nu;
    p.smem = fixed + (size_t)stages * N * 128;
    return p;
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool make_map_bf16(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows) {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * 2)};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_tc_rec(const TcRecArgs& a, cudaStream_t s) {
    const TcRecPlan& p = a.p;
    CUtensorMap tmH, tmW;
    const long long hrows = (long long)a.D * (a.T + 1) * a.B;
    if (!make_map_bf16(&tmH, a.hx, hrows, a.H, p.N)) return cudaErrorInvalidValue;
    if (!make_map_bf16(&tmW, a.wpk, (long long)a.D * 4 * a.H, a.H, kRows)) return cudaErrorInvalidValue;
    TcRecParams prm{};
    prm.H = a.H; prm.B = a.B; prm.T = a.T; prm.D = a.D;
    prm.nbg = p.nbg; prm.Bg = p.Bg; prm.N = p.N; prm.nu = p.nu; prm.kc_smem = p.kc_smem; prm.stages = p.stages;
    prm.gx = a.gx; prm.c0 = a.c0;
    prm.hx = static_cast<bf16*>(a.hx);
    prm.hseq = static_cast<bf16*>(a.hseq);
    prm.out = static_cast<bf16*>(a.out); prm.out_st = a.out_st; prm.out_sb = a.out_sb;
    prm.h_n = static_cast<bf16*>(a.h_n); prm.c_n = a.c_n;
    prm.wpk = static_cast<const bf16*>(a.wpk);
    prm.ctr = a.ctr; prm.status = a.status; prm.timeout_ns = a.timeout_ns;
    cudaError_t e = cudaFuncSetAttribute(tc_rec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return e;
    void* params[] = {&tmH, &tmW, &prm};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(&tc_rec_kernel), dim3(p.ctas), dim3(kThreads),
                                       params, p.smem, s);
}

}  // namespace lstm
