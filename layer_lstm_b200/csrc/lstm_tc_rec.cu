// Persistent LSTM forward recurrence on the sm_100a tensor cores (bf16).
//
// Each step computes, for every direction d, the gate pre-activations
//     a[p][b] = sum_k W_hh[p][k] h_{t-1}[b][k] + Gx[t][b][p]
// (warp_nn "Long Short-Term Memory (LSTM)" equation block; Gx holds
// W_ih x_t + b_ih + b_hh from the time-batched projection) and the cell
// update c = f c + i g, h = o tanh(c).
//
// A cluster of two blocks owns 128 packed gate rows p = 4u + q (units
// [32j, 32j+32)) and the N batch columns of group bg.  The pair splits K:
// block rank r keeps the K chunks [r*KH, r*KH + KH) of the 128-row W_hh slice
// resident for the whole sequence (tensor memory, where tcgen05.mma reads it
// as the A operand; chunks beyond its capacity in shared memory) and issues
// the MMAs of its half only, so the serial chain of MMA instructions per step
// is half as long as with one block per slice.  Each block owns half of the N
// columns: it sends its partial sums of the partner's columns into the
// partner's shared memory (asynchronous distributed-shared-memory stores that
// complete on the partner's mbarrier), adds the partner's partial sums of its
// own columns, and updates c and h there.  One step:
//   warp 0:     wait for the group's h_{t-1}, TMA this block's K chunks of it
//               (N rows x 64 k each) through a ring of shared-memory stages
//   warp 1:     once the accumulator holds Gx[t] in the own columns and zero
//               in the partner's (d_ready), one thread issues M=128 x N x
//               K=16 MMAs over the block's K chunks
//   warps 2-9:  (two per tensor-memory lane quarter) exchange partial sums
//               with the partner, exchange the four gates of each unit inside
//               4-lane groups (shuffles), update c (registers) and h, write
//               h_t and arrive on the group counter; then load Gx[t+1] (L2
//               prefetched one step ahead) into the accumulator and signal
//               d_ready.
// bf16 only.  In training the cells also write the gate activations and cell
// states the backward reads.  Every wait is bounded: on a timeout the kernel
// records LSTM_ERR_TIMEOUT in the status word and returns.
#include <cuda_fp16.h>

#include <algorithm>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"
#include "lstm_tc_cluster.cuh"

namespace lstm {
namespace {

constexpr int kRows = 128;             // gate rows per block
constexpr int kChunkW = kRows * 128;   // bytes of one 64-wide K chunk of W
constexpr int kMaxN = 256;             // batch columns per cluster
constexpr int kCcPerHalf = 4;          // own 16-column chunks per epilogue thread (N/2 <= 128)
constexpr int kEpi = 256;              // epilogue threads: warps 2-9, two per lane quarter
constexpr int kThreads = 64 + kEpi;    // warp 0 TMA, warp 1 MMA
constexpr uint32_t kAcol = 256;        // tensor-memory column of the resident W part
constexpr int kMaxTmemChunks = 8;      // 8 x 32 columns of W in tensor memory
// Shared memory requested per block is at least this, so that two blocks
// never share an SM (each allocates all 512 tensor-memory columns).
constexpr size_t kMinSmem = 120 * 1024;
constexpr int kCtrStride = 32;         // unsigned words between group counters (one 128-byte line each)
constexpr unsigned kFullMask = 0xffffffffu;

struct TcRecParams {
    int H, B, T, D;
    int nbg, Bg, N, nu, KH, kc_smem, stages;
    const float* gx;          // [T][B][D*G] packed rows, biases included
    const float* c0;          // [D][B][H] or null
    bf16* hx;                 // [D][T+1][B][H]; slot 0 holds h0
    bf16* hseq;               // [T][B][D*H] or null
    bf16* out; long long out_st, out_sb;
    int out_vec;              // out is 16-byte aligned: h leaves in 16-byte stores
    bf16* h_n; float* c_n;    // [D][B][H]
    const bf16* wpk;          // [D*G][H] packed rows
    unsigned* ctr;            // [D][nbg] group counters, kCtrStride apart
    int* status;
    uint64_t timeout_ns;
    unsigned long long* trace;   // per-step timeline of block 0, or null
    const int* len;              // [B] valid steps per row, or null (all T)
    float* act;                  // training: [D][T][B][G] gate activations (i, f, g, o of unit u at 4u), or null
    float* cst;                  // training: [D][T][B][H] cell states
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

// Gate nonlinearities of this bf16-only kernel: tanh of two values with one
// special-function op (f16x2: arguments and results rounded to half
// precision, error near 2^-10 -- below the rounding of h to bf16 that this
// path applies every step).
__device__ __forceinline__ float2 tanh2(float a, float b) {
    const __half2 x = __floats2half2_rn(a, b);
    uint32_t r;
    asm("tanh.approx.f16x2 %0, %1;" : "=r"(r) : "r"(*reinterpret_cast<const uint32_t*>(&x)));
    return __half22float2(*reinterpret_cast<const __half2*>(&r));
}

__device__ __forceinline__ float2 sigmoid2(float a, float b) {
    const float2 t = tanh2(0.5f * a, 0.5f * b);
    return make_float2(fmaf(0.5f, t.x, 0.5f), fmaf(0.5f, t.y, 0.5f));
}

// Accumulator initialisation for one step: Gx[t] of packed row `prow` in the
// own columns (chunks cc = half, half + 2, ... of [own0, own0 + NH); zero past
// the batch), zero in the partner's columns; then d_ready.  Two own chunks'
// loads are in flight before their tensor-memory stores.
__device__ __forceinline__ void preload_gx(const float* gx, int t, int B, size_t ldgx, int prow, int b0, int own0,
                                           int pcol0, int ncc, int nB, int half, uint32_t trow, uint64_t* d_ready) {
    const float* gxp = gx + (size_t)t * B * ldgx + (size_t)prow;
    uint32_t zero[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) zero[i] = 0u;
#pragma unroll
    for (int k = 0; k < kCcPerHalf; k += 2) {
        const int cc0 = half + 2 * k, cc1 = cc0 + 2;
        if (cc0 >= ncc) break;
        uint32_t v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int cc = i < 16 ? cc0 : cc1;
            const int col = own0 + 16 * cc + (i & 15);
            v[i] = (cc < ncc && col < nB) ? __float_as_uint(__ldg(gxp + (size_t)(b0 + col) * ldgx)) : 0u;
        }
        uint32_t lo[16], hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) { lo[i] = v[i]; hi[i] = v[16 + i]; }
        tc::tmem_st16(trow + (uint32_t)(own0 + 16 * cc0), lo);
        tc::tmem_st16(trow + (uint32_t)(pcol0 + 16 * cc0), zero);
        if (cc1 < ncc) {
            tc::tmem_st16(trow + (uint32_t)(own0 + 16 * cc1), hi);
            tc::tmem_st16(trow + (uint32_t)(pcol0 + 16 * cc1), zero);
        }
    }
    tc::tmem_st_wait();
    tc::tc_fence_before();
    tc::mbar_arrive(d_ready);
}

// kWsmem: some of the block's W_hh chunks live in shared memory (plans with
// more K chunks than tensor memory holds).  The two operand forms of
// tcgen05.mma are compiled into separate kernels: a loop that can issue
// either form (a branch between them) runs at 120-160 cycles per MMA, a loop
// of one form at the tensor pipe's rate (55 cycles at N = 32, 128 at
// N = 256; measured with the tcgen05.mma issue probe).
// kWhole: the block's whole K share of h_{t-1} fits the stage ring and comes
// in as one 3-D TMA box per step (tmH3), chunk i into stage i; otherwise the
// chunks stream through the ring one 2-D box each (tmH).
// kTrain: the cells also store the gate activations and cell states the
// backward reads (a separate instance, so inference carries none of it).
template <bool kWsmem, bool kWhole, bool kTrain>
__global__ void __launch_bounds__(kThreads, 1)
    tc_rec_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmH3,
                  const __grid_constant__ CUtensorMap tmW, TcRecParams a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int S = a.stages, N = a.N, NH = N / 2;
    const int hstage = N * 128;
    // epilogue column chunks: 8 wide for the small groups of whole-box plans
    // (both halves of the epilogue warps busy at N = 32), else 16
    constexpr int kCW = kWhole ? 8 : 16;
    constexpr int kQW = kCW / 4;   // columns per lane after the gate exchange
    const uint32_t rank = cluster_rank();
    const int KT = H / 64;
    const int c_beg = (int)rank * a.KH, c_end = min(KT, c_beg + a.KH);
    const int nch = c_end - c_beg;                     // K chunks of this block (>= 1)
    const int kc_smem = kWsmem ? min(nch, a.kc_smem) : 0;   // of which in shared memory
    unsigned char* sW = smem;
    unsigned char* sH = smem + a.kc_smem * kChunkW;
    // partner's partial sums of the own columns, [NH/4][128 rows] float4 (a
    // warp's store of one column quad is 512 contiguous bytes)
    float4* recv = reinterpret_cast<float4*>(sH + S * hstage);
    // h of the own columns, [NH][32 units] bf16, 16-byte unit octets swizzled
    bf16* sh = reinterpret_cast<bf16*>(recv + (size_t)(NH / 4) * kRows);
    uint64_t* full = reinterpret_cast<uint64_t*>(sh + (size_t)NH * 32);
    uint64_t* empty = full + S;
    uint64_t* d_ready = empty + S;
    uint64_t* mma_done = d_ready + 1;
    uint64_t* w_full = mma_done + 1;
    uint64_t* recv_full = w_full + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool tr0 = blockIdx.x == 0 && lane == 0;             // traced lane of warps 0 and 1
    const bool tr2 = blockIdx.x == 0 && warp == 2 && lane == 0;   // traced epilogue thread
    const int cl = blockIdx.x >> 1;                    // cluster index; rank == blockIdx.x & 1
    const int j = cl % a.nu;
    const int bg = (cl / a.nu) % a.nbg;
    const int d = cl / (a.nu * a.nbg);
    const int b0 = bg * a.Bg, nB = min(a.Bg, B - b0);
    const int prow0 = d * G + j * kRows;
    const int own0 = (int)rank * NH;                   // first own column
    const int pcol0 = (int)(rank ^ 1u) * NH;           // first column of the partner
    // group counter of (d, bg): every block of the group adds 1 when its h_t
    // columns are out, so h_t is complete at 2 nu (s + 1)
    unsigned* ctr = a.ctr + (size_t)(d * a.nbg + bg) * kCtrStride;
    // K chunks in rotated order, so the blocks of a group spread their reads
    // of h over the chunks
    const int rot = j % nch;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        tc::mbar_init(d_ready, kEpi);
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(w_full, 1);
        tc::mbar_init(recv_full, 1);                  // armed each step with the partner's bytes
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
    cluster_sync();                                    // the partner's barriers exist before any remote arrive
    const uint32_t tmem = *tmem_slot;

    // Resident weights of this block's K chunks: the first kc_smem in shared
    // memory by TMA, the rest in tensor memory (row r of the slice on lane r,
    // two bf16 per column) by the first four epilogue warps.
    if (warp == 0 && lane == 0) {
        tc::prefetch_tmap(kWhole ? &tmH3 : &tmH);
        tc::prefetch_tmap(&tmW);
        if (kc_smem > 0) {
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(kc_smem * kChunkW));
            for (int c = 0; c < kc_smem; ++c) tc::tma_load_2d(sW + c * kChunkW, &tmW, 64 * (c_beg + c), prow0, w_full);
        }
    }
    const int q = warp & 3;                 // lane quarter of an epilogue warp
    const int r = q * 32 + lane;            // accumulator row of this epilogue thread
    const int half = (warp - 2) >> 2;       // 0 or 1 for epilogue warps
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    if (warp >= 2 && half == 0) {
        const bf16* wrow = a.wpk + (size_t)(prow0 + r) * H;
        for (int c = c_beg + kc_smem; c < c_end; ++c) {
            const uint4* src = reinterpret_cast<const uint4*>(wrow + 64 * c);
            uint32_t v0[16], v1[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 x = src[i];
                v0[4 * i] = x.x; v0[4 * i + 1] = x.y; v0[4 * i + 2] = x.z; v0[4 * i + 3] = x.w;
                const uint4 y = src[4 + i];
                v1[4 * i] = y.x; v1[4 * i + 1] = y.y; v1[4 * i + 2] = y.z; v1[4 * i + 3] = y.w;
            }
            const uint32_t col = kAcol + (uint32_t)(c - c_beg - kc_smem) * 32;
            tc::tmem_st16(trow + col, v0);
            tc::tmem_st16(trow + col + 16, v1);
        }
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    // The producer and MMA warps run their loops as whole warps: every lane
    // waits (warp-uniform outcome through a vote), one elected lane issues.
    if (warp == 0) {
        // ------------------------------------------------------ h producer
        int issued = 0;
        bool ok = true;
        for (int s = 0; s < T && ok; ++s) {
            if (s > 0) {
                // the group counter is polled by one lane (a global load, not
                // an mbarrier); __syncwarp orders its acquire before the
                // elected lane's copy
                bool got = true;
                if (lane == 0) got = ctr_wait(ctr, (unsigned)(2 * a.nu * s), abort_flag, a.status, a.timeout_ns);
                got = __shfl_sync(kFullMask, got, 0);
                __syncwarp();
                if (!got) break;
                tc::fence_proxy_async_global();
            }
            trace_mark(a.trace, tr0, s, 0);
            const int row0 = (d * (T + 1) + s) * B + b0;
            if (kWhole) {
                // the whole K share in one box: chunk i into stage i; the
                // ring is free once the previous step's MMAs completed
                if (s > 0 &&
                    !__all_sync(kFullMask, tc::mbar_wait(&empty[0], (s - 1) & 1, abort_flag, a.status, a.timeout_ns)))
                    break;
                if (tc::elect_one()) {
                    tc::mbar_arrive_expect_tx(&full[0], (uint32_t)(a.KH * hstage));
                    tc::tma_load_3d(sH, &tmH3, 0, row0, c_beg, &full[0]);
                }
                __syncwarp();
                ++issued;
                trace_mark(a.trace, tr0, s, 1);
                continue;
            }
            for (int i = 0; i < nch; ++i) {
                const int c = rot + i < nch ? rot + i : rot + i - nch;
                const int st = issued % S, rnd = issued / S;
                if (!__all_sync(kFullMask,
                                tc::mbar_wait(&empty[st], (rnd & 1) ^ 1, abort_flag, a.status, a.timeout_ns))) {
                    ok = false;
                    break;
                }
                if (tc::elect_one()) {
                    tc::mbar_arrive_expect_tx(&full[st], (uint32_t)hstage);
                    tc::tma_load_2d(sH + st * hstage, &tmH, 64 * (c_beg + c), row0, &full[st]);
                }
                __syncwarp();
                ++issued;
            }
            trace_mark(a.trace, tr0, s, 1);
        }
        if (*abort_flag) {
            if (kWhole) {
                if (issued > 0) drain_wait(&full[0], (issued - 1) & 1);
            } else {
                for (int idx = issued > S ? issued - S : 0; idx < issued; ++idx)
                    drain_wait(&full[idx % S], (idx / S) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        // Each elected block issues its MMAs and their commits together, so
        // a commit always follows the MMAs of its own thread.
        const uint32_t idesc = tc::instr_desc(1, kRows, N);
        bool ok = kc_smem == 0 || __all_sync(kFullMask, tc::mbar_wait(w_full, 0, abort_flag, a.status, a.timeout_ns));
        int last = -1;
        for (int s = 0; s < T && ok; ++s) {
            if (!__all_sync(kFullMask, tc::mbar_wait(d_ready, s & 1, abort_flag, a.status, a.timeout_ns))) break;
            tc::tc_fence_after();
            trace_mark(a.trace, tr0, s, 2);
            if (kWhole) {
                if (!__all_sync(kFullMask, tc::mbar_wait(&full[0], s & 1, abort_flag, a.status, a.timeout_ns))) break;
                tc::tc_fence_after();
                trace_mark(a.trace, tr0, s, 9);
                if (tc::elect_one()) {
                    for (int i = 0; i < nch; ++i) {
                        const int c = i;
                        const uint32_t b_base = tc::smem_u32(sH + i * hstage);
                        if (kWsmem && c < kc_smem) {
                            const uint32_t a_base = tc::smem_u32(sW + c * kChunkW);
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj)
                                tc::mma_bf16(tmem, tc::smem_desc_sw128(a_base + 32 * jj),
                                             tc::smem_desc_sw128(b_base + 32 * jj), idesc, 1);
                        } else {
                            const uint32_t at = tmem + kAcol + (uint32_t)(c - kc_smem) * 32;
#pragma unroll
                            for (int jj = 0; jj < 4; ++jj)
                                tc::mma_bf16_ts(tmem, at + 8 * jj, tc::smem_desc_sw128(b_base + 32 * jj), idesc, 1);
                        }
                    }
                    tc::mma_commit(&empty[0]);
                    tc::mma_commit(mma_done);
                }
                __syncwarp();
                last = s;
                trace_mark(a.trace, tr0, s, 3);
                continue;
            }
            for (int i = 0; i < nch; ++i) {
                const int idx = s * nch + i, st = idx % S, rnd = idx / S;
                if (!__all_sync(kFullMask, tc::mbar_wait(&full[st], rnd & 1, abort_flag, a.status, a.timeout_ns))) {
                    ok = false;
                    break;
                }
                tc::tc_fence_after();
                const int c = rot + i < nch ? rot + i : rot + i - nch;
                if (i == 0) trace_mark(a.trace, tr0, s, 9);
                const uint32_t b_base = tc::smem_u32(sH + st * hstage);
                if (tc::elect_one()) {
                    if (kWsmem && c < kc_smem) {
                        const uint32_t a_base = tc::smem_u32(sW + c * kChunkW);
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            tc::mma_bf16(tmem, tc::smem_desc_sw128(a_base + 32 * jj),
                                         tc::smem_desc_sw128(b_base + 32 * jj), idesc, 1);
                    } else {
                        const uint32_t at = tmem + kAcol + (uint32_t)(c - kc_smem) * 32;
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj)
                            tc::mma_bf16_ts(tmem, at + 8 * jj, tc::smem_desc_sw128(b_base + 32 * jj), idesc, 1);
                    }
                    tc::mma_commit(&empty[st]);
                    if (i == nch - 1) tc::mma_commit(mma_done);
                }
                __syncwarp();
                last = idx;
            }
            if (!ok) break;
            trace_mark(a.trace, tr0, s, 3);
        }
        if (*abort_flag && last >= 0) {
            if (kWhole)
                drain_wait(&empty[0], last & 1);
            else
                drain_wait(&empty[last % S], (last / S) & 1);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int e = threadIdx.x - 64;             // epilogue thread index
        const int gq = lane & 3;                    // gate of this lane's row
        const int u = j * 32 + q * 8 + (lane >> 2); // unit of this lane's row group
        const int ncc = NH / kCW;                   // own column chunks
        const int ncc16 = NH / 16;                  // own 16-column chunks (the Gx preload's unit)
        const uint32_t partner = rank ^ 1u;
        const uint32_t recv_remote = map_rank(tc::smem_u32(recv), partner);
        const uint32_t recv_bar_remote = map_rank(tc::smem_u32(recv_full), partner);
        const size_t ldgx = (size_t)D * G;
        const size_t ldseq = (size_t)D * H;
        float creg[kCcPerHalf][4];
#pragma unroll
        for (int k = 0; k < kCcPerHalf; ++k)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cc = half + 2 * k;
                const int col = own0 + kCW * cc + kQW * gq + i;
                creg[k][i] = (i < kQW && cc < ncc && col < nB && a.c0) ? a.c0[((size_t)d * B + b0 + col) * H + u]
                                                                       : 0.f;
            }
        preload_gx(a.gx, d == 0 ? 0 : T - 1, B, ldgx, prow0 + r, b0, own0, pcol0, ncc16, nB, half, trow, d_ready);
        for (int s = 0; s < T; ++s) {
            const int t = d == 0 ? s : T - 1 - s;
            // this step's phase of recv_full completes when the partner's
            // partial sums of the own columns (NH x 128 floats) have landed;
            // the previous phase completed before this thread left step s-1
            if (e == 0) tc::mbar_arrive_expect_tx(recv_full, (uint32_t)(NH * kRows * 4));
            // Gx[t_next] of the own columns into L2 while the MMAs run
            if (s + 1 < T && e < NH && own0 + e < nB) {
                const int tn = d == 0 ? s + 1 : T - 2 - s;
                prefetch_l2(a.gx + ((size_t)tn * B + b0 + own0 + e) * ldgx + prow0, kRows * 4);
            }
            const bool ok = tc::mbar_wait(mma_done, s & 1, abort_flag, a.status, a.timeout_ns);
            if (tc::named_bar_or(1, kEpi, !ok)) break;   // every epilogue thread leaves together
            tc::tc_fence_after();
            trace_mark(a.trace, tr2, s, 4);
            // 1) this block's partial sums of the partner's columns -> partner,
            //    two column chunks at a time (recv holds column quads)
#pragma unroll
            for (int k0 = 0; k0 < kCcPerHalf; k0 += 2) {
                if (half + 2 * k0 >= ncc) break;
                float pv[2][kCW];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int cc = half + 2 * (k0 + kk);
                    if (cc < ncc) tc::tmem_ldw<kCW>(trow + (uint32_t)(pcol0 + kCW * cc), pv[kk]);
                }
                tc::tmem_ld_wait();
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int cc = half + 2 * (k0 + kk);
                    if (cc >= ncc) break;
#pragma unroll
                    for (int m = 0; m < kCW / 4; ++m)
                        st_async_v4(recv_remote + (uint32_t)((((kCW / 4) * cc + m) * kRows + r) * 16), pv[kk][4 * m],
                                    pv[kk][4 * m + 1], pv[kk][4 * m + 2], pv[kk][4 * m + 3], recv_bar_remote);
                }
            }
            trace_mark(a.trace, tr2, s, 5);
            // 2) the partner's partial sums of the own columns
            const bool got = mbar_wait_cluster(recv_full, s & 1, abort_flag, a.status, a.timeout_ns);
            if (tc::named_bar_or(1, kEpi, !got)) break;
            trace_mark(a.trace, tr2, s, 6);
            // 3) gates, cell update and h for the own columns, two chunks at a time
#pragma unroll
            for (int k0 = 0; k0 < kCcPerHalf; k0 += 2) {
                if (half + 2 * k0 >= ncc) break;
                float ov[2][kCW];
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int cc = half + 2 * (k0 + kk);
                    if (cc < ncc) tc::tmem_ldw<kCW>(trow + (uint32_t)(own0 + kCW * cc), ov[kk]);
                }
                tc::tmem_ld_wait();
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int k = k0 + kk;
                    const int cc = half + 2 * k;
                    if (cc >= ncc) break;
                    float* v = ov[kk];
#pragma unroll
                    for (int m = 0; m < kCW / 4; ++m) {
                        const float4 p4 = recv[((kCW / 4) * cc + m) * kRows + r];
                        v[4 * m] += p4.x; v[4 * m + 1] += p4.y; v[4 * m + 2] += p4.z; v[4 * m + 3] += p4.w;
                    }
                    // v[kQW m + i]: gate gq at column kCW cc + kQW m + i.  Three
                    // xor exchanges inside each 4-lane group give lane gq all
                    // four gates at column kCW cc + kQW gq + i (gate X arrives in
                    // round gq ^ X).
                    float gi[kQW], gf[kQW], gc[kQW], go[kQW];
#pragma unroll
                    for (int i = 0; i < kQW; ++i) {
                        float rcv[4];
                        rcv[0] = sel4(v[i], v[kQW + i], v[2 * kQW + i], v[3 * kQW + i], gq);
#pragma unroll
                        for (int rr = 1; rr < 4; ++rr)
                            rcv[rr] = __shfl_xor_sync(
                                0xffffffffu, sel4(v[i], v[kQW + i], v[2 * kQW + i], v[3 * kQW + i], gq ^ rr), rr);
                        gi[i] = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 0);
                        gf[i] = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 1);
                        gc[i] = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 2);
                        go[i] = sel4(rcv[0], rcv[1], rcv[2], rcv[3], gq ^ 3);
                    }
                    // the cells of two columns at a time: every nonlinearity
                    // is one f16x2 tanh for both
#pragma unroll
                    for (int i = 0; i < kQW; i += 2) {
                        const float2 ig = sigmoid2(gi[i], gi[i + 1]), fg = sigmoid2(gf[i], gf[i + 1]);
                        const float2 og = sigmoid2(go[i], go[i + 1]), gg = tanh2(gc[i], gc[i + 1]);
                        const float cn0 = fg.x * creg[k][i] + ig.x * gg.x;
                        const float cn1 = fg.y * creg[k][i + 1] + ig.y * gg.y;
                        const float2 tcn = tanh2(cn0, cn1);
                        const float hn[2] = {og.x * tcn.x, og.y * tcn.y};
                        const float cn[2] = {cn0, cn1};
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int lc = kCW * cc + kQW * gq + i + e;   // column within the own half
                            const int col = own0 + lc;
                            if (col >= nB) continue;
                            const int bb = b0 + col;
                            bf16 hv;
                            float c = creg[k][i + e];
                            const bool valid = !a.len || t < a.len[bb];
                            if (valid) {
                                c = cn[e];
                                creg[k][i + e] = c;
                                hv = __float2bfloat16_rn(hn[e]);
                            } else {
                                // padding of a variable-length row: the state stays
                                hv = __ldcg(a.hx + ((size_t)(d * (T + 1) + s) * B + bb) * H + u);
                            }
                            if (kTrain) {   // what the backward reads (zero gates at padding)
                                const size_t row = ((size_t)d * T + t) * B + bb;
                                *reinterpret_cast<float4*>(a.act + row * G + 4 * u) =
                                    valid ? make_float4(e ? ig.y : ig.x, e ? fg.y : fg.x, e ? gg.y : gg.x,
                                                        e ? og.y : og.x)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
                                a.cst[row * H + u] = c;
                            }
                            // unit octet q of column lc, stored at octet
                            // q ^ ((lc >> 2) & 3) (= gq with 16-column chunks):
                            // the columns of a warp's store fall in different banks
                            sh[lc * 32 + 8 * (q ^ ((lc >> 2) & 3)) + (lane >> 2)] = hv;
                            if (s == T - 1) {
                                const int b = b0 + col;
                                a.h_n[((size_t)d * B + b) * H + u] = hv;
                                a.c_n[((size_t)d * B + b) * H + u] = c;
                            }
                        }
                    }
                }
            }
            trace_mark(a.trace, tr2, s, 7);
            // 4) h_t of the own columns to global memory in 16-byte pieces
            //    (32 units of a column are 64 contiguous bytes), publish it
            //    to the group, then hand the accumulator Gx[t+1]
            tc::named_bar_sync(1, kEpi);
            {
                bf16* hxo = a.hx + ((size_t)(d * (T + 1) + s + 1) * B) * H + 32 * j;
                for (int idx = e; idx < NH * 4; idx += kEpi) {
                    const int lc = idx >> 2, oct = idx & 3;
                    if (own0 + lc >= nB) continue;
                    const int b = b0 + own0 + lc;
                    const uint4 val = *reinterpret_cast<const uint4*>(sh + lc * 32 + 8 * (oct ^ ((lc >> 2) & 3)));
                    *reinterpret_cast<uint4*>(hxo + (size_t)b * H + 8 * oct) = val;
                }
            }
            tc::fence_proxy_async_global();
            tc::named_bar_sync(1, kEpi);
            if (warp == 2 && lane == 0) {
                red_release_add(ctr, 1u);
            }
            trace_mark(a.trace, tr2, s, 8);
            if (s + 1 < T) {
                preload_gx(a.gx, d == 0 ? s + 1 : T - 2 - s, B, ldgx, prow0 + r, b0, own0, pcol0, ncc16, nB, half, trow,
                           d_ready);
                trace_mark(a.trace, tr2, s + 1, 10);
            }
            // the layer output and the user output leave after the release
            // and the accumulator hand-over: the group's next step waits only
            // for the exchange copy
            {
                for (int idx = e; idx < NH * 4; idx += kEpi) {
                    const int lc = idx >> 2, oct = idx & 3;
                    if (own0 + lc >= nB) continue;
                    const int b = b0 + own0 + lc;
                    const uint4 val = *reinterpret_cast<const uint4*>(sh + lc * 32 + 8 * (oct ^ ((lc >> 2) & 3)));
                    const size_t uo = (size_t)d * H + 32 * j + 8 * oct;
                    if (a.hseq) *reinterpret_cast<uint4*>(a.hseq + ((size_t)t * B + b) * ldseq + uo) = val;
                    if (a.out && a.len && t >= a.len[b]) {   // padding: the user output is 0
                        bf16* dst = a.out + (size_t)t * a.out_st + (size_t)b * a.out_sb + uo;
#pragma unroll
                        for (int x = 0; x < 8; ++x) dst[x] = __float2bfloat16_rn(0.f);
                    } else if (a.out) {
                        bf16* dst = a.out + (size_t)t * a.out_st + (size_t)b * a.out_sb + uo;
                        if (a.out_vec) {
                            *reinterpret_cast<uint4*>(dst) = val;
                        } else {
                            const bf16* sv = reinterpret_cast<const bf16*>(&val);
#pragma unroll
                            for (int x = 0; x < 8; ++x) dst[x] = sv[x];
                        }
                    }
                }
            }

        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
    cluster_sync();   // neither block leaves while its partner may still write into it
}

}  // namespace

TcRecPlan plan_tc_rec(int H, int B, int D, int num_sms, size_t smem_max) {
    TcRecPlan p{};
    if (H % 64 != 0 || H < 128 || B < 1) return p;
    const int KT = H / 64;
    const int KH = (KT + 1) / 2;                      // K chunks of the first block of a pair
    const int nu = 4 * H / kRows;
    const int kc_smem = std::max(0, KH - kMaxTmemChunks);
    const int max_groups = num_sms / (2 * D * nu);
    if (max_groups < 1) return p;
    int nbg = std::min(max_groups, std::max(1, (B + 31) / 32));
    int Bg = (B + nbg - 1) / nbg;
    while (((Bg + 31) / 32) * 32 > kMaxN && nbg < max_groups) {
        ++nbg;
        Bg = (B + nbg - 1) / nbg;
    }
    const int N = ((Bg + 31) / 32) * 32;               // two halves of whole 16-column chunks
    if (N > kMaxN) return p;
    if (nbg > 1 && (nbg - 1) * Bg >= B) return p;
    const size_t recv = (size_t)kRows * (N / 2) * 4 + (size_t)(N / 2) * 32 * 2;   // partial sums, h staging
    const size_t fixed = (size_t)kc_smem * kChunkW + recv + 1024 + 256;
    int stages = 8;
    while (stages >= 2 && fixed + (size_t)stages * N * 128 > smem_max) --stages;
    if (stages < 2) return p;
    p.ok = true;
    p.nbg = nbg; p.Bg = Bg; p.N = N; p.nu = nu; p.KH = KH; p.kc_smem = kc_smem; p.stages = stages;
    p.ctas = 2 * D * nbg * nu;
    p.smem = std::min(smem_max, std::max(kMinSmem, fixed + (size_t)stages * N * 128));
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

// h_{t-1} as a 3-D tensor (k within a 64-wide chunk, row, chunk): a box of
// {64, rows, chunks} lands the chunks one after another, each a 128-byte-
// swizzled [rows][64] tile, as the 2-D boxes of single chunks would.
bool make_map_bf16_chunks(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows,
                          int box_chunks) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return false;
    const EncodeTiledFn fn = reinterpret_cast<EncodeTiledFn>(p);
    cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(cols / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)(cols * 2), 128};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)box_chunks};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_tc_rec(const TcRecArgs& a, cudaStream_t s) {
    const TcRecPlan& p = a.p;
    CUtensorMap tmH, tmH3, tmW;
    const long long hrows = (long long)a.D * (a.T + 1) * a.B;
    if (!make_map_bf16(&tmH, a.hx, hrows, a.H, p.N)) return cudaErrorInvalidValue;
    // one box per step when both blocks of a pair hold KH chunks and the
    // ring holds them all
    const int KT = a.H / 64;
    const bool whole = KT % 2 == 0 && p.stages >= p.KH && p.KH <= 256 &&
                       make_map_bf16_chunks(&tmH3, a.hx, hrows, a.H, p.N, p.KH);
    if (!whole) tmH3 = tmH;
    if (!make_map_bf16(&tmW, a.wpk, (long long)a.D * 4 * a.H, a.H, kRows)) return cudaErrorInvalidValue;
    TcRecParams prm{};
    prm.H = a.H; prm.B = a.B; prm.T = a.T; prm.D = a.D;
    prm.nbg = p.nbg; prm.Bg = p.Bg; prm.N = p.N; prm.nu = p.nu; prm.KH = p.KH;
    prm.kc_smem = p.kc_smem; prm.stages = p.stages;
    prm.gx = a.gx; prm.c0 = a.c0;
    prm.hx = static_cast<bf16*>(a.hx);
    prm.hseq = static_cast<bf16*>(a.hseq);
    prm.out = static_cast<bf16*>(a.out); prm.out_st = a.out_st; prm.out_sb = a.out_sb;
    prm.out_vec = (reinterpret_cast<uintptr_t>(a.out) & 15) == 0;
    prm.h_n = static_cast<bf16*>(a.h_n); prm.c_n = a.c_n;
    prm.wpk = static_cast<const bf16*>(a.wpk);
    prm.trace = a.trace;
    prm.len = a.len;
    prm.ctr = a.ctr; prm.status = a.status; prm.timeout_ns = a.timeout_ns;
    prm.act = a.act; prm.cst = a.cst;
    // one operand form per kernel: tensor memory only, unless chunks spill
    // to shared memory
    const bool train = a.act != nullptr;
    using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, TcRecParams);
    static const Kern kTable[8] = {tc_rec_kernel<false, false, false>, tc_rec_kernel<false, false, true>,
                                   tc_rec_kernel<false, true, false>,  tc_rec_kernel<false, true, true>,
                                   tc_rec_kernel<true, false, false>,  tc_rec_kernel<true, false, true>,
                                   tc_rec_kernel<true, true, false>,   tc_rec_kernel<true, true, true>};
    const auto kern = kTable[(p.kc_smem > 0 ? 4 : 0) + (whole ? 2 : 0) + (train ? 1 : 0)];
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Every block waits on the others of its group, so the whole grid must be
    // resident at once: the launch is refused unless the device can hold all
    // its clusters together.  The launch carries no cooperative attribute
    // (cluster launches with it failed under the profiler); should the grid
    // not be co-scheduled all the same, the bounded waits end the call with
    // LSTM_ERR_TIMEOUT instead of a hang.
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (2 * clusters < p.ctas) return cudaErrorCooperativeLaunchTooLarge;
    return cudaLaunchKernelEx(&cfg, kern, tmH, tmH3, tmW, prm);
}

}  // namespace lstm
