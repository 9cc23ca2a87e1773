// Persistent LSTM forward recurrence on the sm_100a tensor cores for float32
// problems: the recurrent product in 3xTF32.
//
// Each step computes, for every direction d, the gate pre-activations
//     a[p][b] = sum_k W_hh[p][k] h_{t-1}[b][k] + Gx[t][b][p]
// and the cell update (warp_nn "Long Short-Term Memory (LSTM)" equation
// block) in float32.  The product runs as kind::tf32 MMAs on operands split
// into a tf32 part and the float32 remainder (x = hi + lo):
//     W h ~= W_hi h_hi + W_hi h_lo + W_lo h_hi,
// the lo*lo term (relative size 2^-22) dropped; sums are float32.
//
// A cluster of C = H/128 blocks owns 128 packed gate rows p = 4u+q (units
// [32j, 32j+32)) and the N batch columns of one group; in tensor memory they
// are gate-major (lane 32q + u - 32j holds gate q of unit u), so a warp's
// accumulator rows are one gate of 32 units.  Block rank r keeps
// the K part [r*KP, r*KP + KP) (KP = H/C <= 128) of those rows resident in
// tensor memory, hi and lo side by side (the A operand of tcgen05.mma), and
// owns the columns [r*N/C, (r+1)*N/C).  Per step:
//   warp 0:    wait for the group's h_{t-1}, TMA the block's K part of it,
//              hi and lo, in kSeg K segments (3-D boxes, 128-byte swizzle)
//              completing on a barrier each, so the MMAs of the first
//              segment run while the next lands
//   warps 1-3: one product each (hi*hi, hi*lo, lo*hi), an MMA per k-step
//              of 8 into an accumulator of its own: three issuing threads
//              keep the tensor pipe busy at N <= 64, where one issues an
//              MMA only every ~55 cycles
//   warps 4-11: add the three accumulators and send each column quad's partial sums to the block that owns
//              the column (asynchronous distributed-shared-memory stores
//              completing on the owner's mbarrier); as owner, add the C
//              partials of each (unit, column) cell and Gx[t], the gates and
//              the cell update, write h_t (split hi | lo) to the exchange and
//              the outputs (and in training the gate activations and cell
//              states), and arrive on the group counter.
// Every wait is bounded: on a timeout the kernel records LSTM_ERR_TIMEOUT.
#include <algorithm>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"
#include "lstm_tc_cluster.cuh"

namespace lstm {
namespace {

constexpr int kRows = 128;                // packed gate rows per slice (MMA M)
constexpr int kEpi = 256;                 // epilogue threads, warps 4-11
constexpr int kIss = 3;                   // issuing warps, one per product
constexpr int kThreads = 32 * (1 + kIss) + kEpi;
constexpr int kMaxN = 64;                 // batch columns per group
constexpr int kMaxCells = 32 * kMaxN / 2 / kEpi;   // cells per epilogue thread (N/C <= 32)
constexpr uint32_t kAcol = 256;           // tensor-memory column of the resident W_hh part (hi, then lo)
static_assert(kIss * kMaxN <= (int)kAcol, "the accumulators fit below the resident W_hh part");
constexpr int kMaxKP = 128;               // K part per block: hi + lo fill the 256 columns
constexpr int kMaxC = 8;                  // blocks per cluster (H <= 1024)
constexpr int kSeg = 2;                   // K segments of a step's h tiles, each on its own barrier
constexpr size_t kMinSmem = 120 * 1024;   // two blocks never share an SM (512 TMEM columns each)
constexpr int kCtrStride = 32;
constexpr unsigned kFullMask = 0xffffffffu;

struct TcRec32Params {
    int H, B, T, D;
    int nbg, Bg, N, nsl, C, KP;
    int d0;                    // first direction of this launch
    const float* gx;
    const float* wpk;          // packed rows 4u+q, or null: W_hh of each direction as given
    const float* w[2];
    const float* c0;
    float* hx;
    float* hseq;
    float* out; long long out_st, out_sb;
    float* h_n; float* c_n;
    float* act; float* cst;
    unsigned* ctr;
    int* status;
    uint64_t timeout_ns;
    const int* len;
    unsigned long long* trace;   // per-step timeline of block 0, or null
    int skip_block, skip_step;   // fault injection (tests of the bounded waits), -1: none
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

__device__ __forceinline__ float sigmoid_f(float z) { return 1.0f / (1.0f + expf(-z)); }

// Exchange slot 0 from h0 (float32 [D][B][H]) or zeros: hi | lo per row.
// One block per (d, b) row, its threads over the row's units.
__global__ void rec32_slot0_kernel(const float* h0, float* hx, int D, int T, int B, int H) {
    for (int db = blockIdx.x; db < D * B; db += gridDim.x) {
        const int d = db / B, b = db - d * B;
        float* row = hx + ((size_t)d * (T + 1) * B + b) * 2 * H;
        for (int u = threadIdx.x; u < H; u += blockDim.x) {
            const float h = h0 ? h0[(size_t)db * H + u] : 0.f;
            const float hi = tf32_hi(h);
            row[u] = hi;
            row[H + u] = h - hi;
        }
    }
}

template <bool kTrain>
__global__ void __launch_bounds__(kThreads, 1)
    tc_rec32_kernel(const __grid_constant__ CUtensorMap tmX, TcRec32Params a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int N = a.N, C = a.C, KP = a.KP, NO = N / C;
    const int nkc = KP / 32;                              // 32-wide K chunks of the part
    const int tile = N * 128;                             // one chunk of h: N rows x 32 floats
    unsigned char* sBh = smem;                            // [nkc][N][32] hi, 128-byte swizzle
    unsigned char* sBl = smem + nkc * tile;               // the same for lo
    // partial sums of the own columns from the C blocks: [src][NO/4 column
    // quads][128 lanes] float4 (4 columns of one gate row)
    float4* recv = reinterpret_cast<float4*>(sBl + nkc * tile);
    uint64_t* full = reinterpret_cast<uint64_t*>(recv + (size_t)C * (NO / 4) * kRows);   // [kSeg]
    uint64_t* empty = full + kSeg;
    uint64_t* d_ready = empty + 1;     // the accumulator was read (count kEpi)
    uint64_t* mma_done = d_ready + 1;
    uint64_t* recv_full = mma_done + 1;
    uint64_t* fin = recv_full + 1;     // [kIss] an issuer's own MMAs drained (abort path)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + kIss);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / C;
    const int j = cl % a.nsl;
    const int bg = (cl / a.nsl) % a.nbg;
    const int d = a.d0 + cl / (a.nsl * a.nbg);
    const int b0 = bg * a.Bg, nB = min(a.Bg, B - b0);
    const int prow0 = d * G + j * kRows;                  // first packed gate row of the slice
    const int kbeg = (int)rank * KP;                      // first k of the part
    const int own0 = (int)rank * NO;                      // first own column
    const int nblk = a.nsl * C;                           // blocks of the (d, bg) group
    unsigned* ctr = a.ctr + (size_t)(d * a.nbg + bg) * kCtrStride;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool tr0 = blockIdx.x == 0 && lane == 0 && warp <= 1;              // producer, first issuer
    const bool tre = blockIdx.x == 0 && warp == 1 + kIss && lane == 0;       // an epilogue thread

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSeg; ++i) tc::mbar_init(full + i, 1);
        tc::mbar_init(empty, kIss);    // one commit per issuer
        tc::mbar_init(d_ready, kEpi);
        tc::mbar_init(mma_done, kIss);
        for (int i = 0; i < kIss; ++i) tc::mbar_init(fin + i, 1);
        tc::mbar_init(recv_full, 1);   // armed each step with the C blocks' bytes
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
    cluster_sync();   // every block's barriers exist before any remote arrive
    const uint32_t tmem = *tmem_slot;

    const int q = warp & 3;                  // lane quarter of an epilogue warp
    const int half = (warp - 1 - kIss) >> 2; // 0 or 1 for epilogue warps
    const int r = q * 32 + lane;             // accumulator row of this thread
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    // Resident W_hh part: gate r / 32 of unit 32j + r % 32 on lane r, one
    // tf32 per column; hi at columns kAcol + k, the remainder at kAcol + KP + k.
    if (warp == 0 && lane == 0) tc::prefetch_tmap(&tmX);
    if (warp > kIss && half == 0) {
        // gate r / 32 of unit 32j + r % 32: packed row 4u + q, or row q*H + u of W_hh as given
        const float* wrow = a.wpk ? a.wpk + (size_t)(prow0 + 4 * (r & 31) + (r >> 5)) * H + kbeg
                                  : a.w[d] + ((size_t)(r >> 5) * H + 32 * j + (r & 31)) * H + kbeg;
        for (int c = 0; c < nkc; ++c) {
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                uint32_t vh[16], vl[16];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 w4 = *reinterpret_cast<const float4*>(wrow + 32 * c + 16 * h16 + 4 * i);
                    const float w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float hi = tf32_hi(w[x]);
                        vh[4 * i + x] = __float_as_uint(hi);
                        vl[4 * i + x] = __float_as_uint(w[x] - hi);
                    }
                }
                tc::tmem_st16(trow + kAcol + (uint32_t)(32 * c + 16 * h16), vh);
                tc::tmem_st16(trow + kAcol + (uint32_t)(KP + 32 * c + 16 * h16), vl);
            }
        }
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    if (warp == 0) {
        // ------------------------------------------------------ h producer
        int issued = 0;
        for (int s = 0; s < T; ++s) {
            if (s > 0) {
                // h_{t-1} is complete when every block of the group arrived s times
                bool got = true;
                if (lane == 0) got = ctr_wait(ctr, (unsigned)(nblk * s), abort_flag, a.status, a.timeout_ns);
                got = __shfl_sync(kFullMask, got, 0);
                __syncwarp();
                if (!got) break;
                tc::fence_proxy_async_global();
                // the tiles are free once the previous step's MMAs completed
                if (!__all_sync(kFullMask, tc::mbar_wait(empty, (s - 1) & 1, abort_flag, a.status, a.timeout_ns)))
                    break;
            }
            trace_mark(a.trace, tr0, s, 0);
            if (tc::elect_one()) {
                const int row0 = (d * (T + 1) + s) * B + b0;
                const int cps = nkc / kSeg;   // chunks per segment
                for (int sg = 0; sg < kSeg; ++sg) {
                    tc::mbar_arrive_expect_tx(full + sg, (uint32_t)(2 * cps * tile));
                    tc::tma_load_3d(sBh + sg * cps * tile, &tmX, 0, row0, kbeg / 32 + sg * cps, full + sg);
                    tc::tma_load_3d(sBl + sg * cps * tile, &tmX, 0, row0, (H + kbeg) / 32 + sg * cps, full + sg);
                }
            }
            __syncwarp();
            ++issued;
        }
        if (*abort_flag && issued > 0)
            for (int sg = 0; sg < kSeg; ++sg) drain_wait(full + sg, (issued - 1) & 1);
    } else if (warp <= kIss) {
        // ------------------------------------------------------------ MMA
        // product pr: A = W_hi (pr < 2) or W_lo, B = h_hi (pr != 1) or h_lo,
        // into the accumulator at column pr * N
        const int pr = warp - 1;
        const uint32_t idesc = tc::instr_desc(2, kRows, N);   // kind::tf32
        const uint32_t acc = tmem + (uint32_t)(pr * N);
        const uint32_t aoff = pr == 2 ? (uint32_t)KP : 0u;
        const unsigned char* sB = pr == 1 ? sBl : sBh;
        int last = -1;
        for (int s = 0; s < T; ++s) {
            if (!__all_sync(kFullMask, tc::mbar_wait(d_ready, s & 1, abort_flag, a.status, a.timeout_ns))) break;
            tc::tc_fence_after();
            last = s;   // from here MMAs of step s may be in flight (drained on abort)
            bool ok = true;
            const int cps = nkc / kSeg;
            for (int sg = 0; sg < kSeg && ok; ++sg) {
                ok = __all_sync(kFullMask, tc::mbar_wait(full + sg, s & 1, abort_flag, a.status, a.timeout_ns));
                if (!ok) break;
                tc::tc_fence_after();
                if (sg == 0) trace_mark(a.trace, tr0, s, 9);
                if (tc::elect_one()) {
                    for (int c = sg * cps; c < (sg + 1) * cps; ++c) {
                        const uint32_t b = tc::smem_u32(sB + c * tile);
#pragma unroll
                        for (int jj = 0; jj < 4; ++jj) {   // k-steps of 8 tf32 (32 bytes of a 128-byte row)
                            const uint32_t aa = tmem + kAcol + aoff + (uint32_t)(32 * c + 8 * jj);
                            tc::mma_tf32_ts(acc, aa, tc::smem_desc_sw128(b + 32 * jj), idesc,
                                            (c | jj) != 0);   // fresh accumulator each step
                        }
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
            if (tc::elect_one()) {
                tc::mma_commit(empty);
                tc::mma_commit(mma_done);
            }
            __syncwarp();
            trace_mark(a.trace, tr0, s, 3);
        }
        if (*abort_flag && last >= 0) {
            // the other issuers may have stopped a step earlier: wait for this
            // thread's own MMAs alone
            if (tc::elect_one()) tc::mma_commit(fin + pr);
            __syncwarp();
            drain_wait(fin + pr, 0);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int e = threadIdx.x - 32 * (1 + kIss);
        const int colh = half * (N / 2);   // sender: row r, columns [colh, colh + N/2)
        const uint32_t recv_s = tc::smem_u32(recv), bar_s = tc::smem_u32(recv_full);
        // owner: cells (unit 32j + (idx >> 2) % 32, own column 4 (idx >> 7) + idx % 4),
        // idx = e + kEpi k: a warp's cells are 8 units of 4 columns
        const int ncell = 32 * NO;
        const size_t ldgx = (size_t)D * G, ldseq = (size_t)D * H;
        float creg[kMaxCells], hreg[kMaxCells];
#pragma unroll
        for (int k = 0; k < kMaxCells; ++k) {
            creg[k] = hreg[k] = 0.f;
            const int idx = e + kEpi * k;
            if (idx >= ncell) continue;
            const int col = own0 + 4 * (idx >> 7) + (idx & 3);
            if (col >= nB) continue;
            const int u = 32 * j + ((idx >> 2) & 31);
            const size_t sidx = ((size_t)d * B + b0 + col) * H + u;
            if (a.c0) creg[k] = a.c0[sidx];
            const float* h0row = a.hx + ((size_t)d * (T + 1) * B + b0 + col) * 2 * H;   // slot 0: h0 = hi + lo
            hreg[k] = h0row[u] + h0row[H + u];
        }
        tc::tc_fence_before();
        tc::mbar_arrive(d_ready);   // the accumulator is free for the first MMAs
        bool stop = false;
        for (int s = 0; s < T && !stop; ++s) {
            const int t = d == 0 ? s : T - 1 - s;
            if (e == 0) tc::mbar_arrive_expect_tx(recv_full, (uint32_t)(C * kRows * NO * 4));
            float4 gxv[kMaxCells];   // Gx[t] of the own cells, fetched before the waits
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                gxv[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                const int idx = e + kEpi * k;
                if (idx >= ncell) continue;
                const int col = own0 + 4 * (idx >> 7) + (idx & 3);
                if (col >= nB) continue;
                gxv[k] = *reinterpret_cast<const float4*>(a.gx + ((size_t)t * B + b0 + col) * ldgx + prow0 +
                                                           4 * ((idx >> 2) & 31));
            }
            const bool ok = tc::mbar_wait(mma_done, s & 1, abort_flag, a.status, a.timeout_ns);
            if (tc::named_bar_or(1, kEpi, !ok)) {
                stop = true;
                break;
            }
            tc::tc_fence_after();
            trace_mark(a.trace, tre, s, 4);
            // row r's partial sums of this half's columns -> the owners' recv[rank]
            for (int c16 = 0; c16 < N / 32; ++c16) {
                float v[16], v1[16], v2[16];
                const int col = colh + 16 * c16;
                tc::tmem_ld16(trow + (uint32_t)col, v);
                tc::tmem_ld16(trow + (uint32_t)(N + col), v1);
                tc::tmem_ld16(trow + (uint32_t)(2 * N + col), v2);
                tc::tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] += v1[i] + v2[i];   // small cross terms first
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int quad = col / 4 + m;
                    const uint32_t o = (uint32_t)(quad * 4 / NO);
                    const int qo = quad - (int)o * (NO / 4);
                    st_async_v4(map_rank(recv_s, o) + (uint32_t)((((int)rank * (NO / 4) + qo) * kRows + r) * 16),
                                v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3], map_rank(bar_s, o));
                }
            }
            tc::tc_fence_before();
            tc::mbar_arrive(d_ready);   // read: the next MMAs may overwrite the accumulator
            trace_mark(a.trace, tre, s, 5);
            const bool got = mbar_wait_cluster(recv_full, s & 1, abort_flag, a.status, a.timeout_ns);
            if (tc::named_bar_or(1, kEpi, !got)) {
                stop = true;
                break;
            }
            trace_mark(a.trace, tre, s, 6);
            // cells: the C partial sums of each gate (fixed order) + Gx[t]
            float* hxo = a.hx + ((size_t)(d * (T + 1) + s + 1) * B) * 2 * H;
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int idx = e + kEpi * k;
                if (idx >= ncell) continue;
                const int ul = (idx >> 2) & 31, clc = 4 * (idx >> 7) + (idx & 3);
                const int col = own0 + clc;
                if (col >= nB) continue;
                const int bb = b0 + col, u = 32 * j + ul;
                const float gx4[4] = {gxv[k].x, gxv[k].y, gxv[k].z, gxv[k].w};
                // (src, quad, lane 32g + ul) holds columns 4 quad .. 4 quad + 3
                const float* rq = reinterpret_cast<const float*>(recv) + ((size_t)(idx >> 7) * kRows + ul) * 4 +
                                  (idx & 3);
                float pre[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int src = 0; src < kMaxC; ++src) {   // independent loads, unrolled
                    if (src >= C) break;
#pragma unroll
                    for (int g = 0; g < 4; ++g) pre[g] += rq[((size_t)src * (NO / 4) * kRows + 32 * g) * 4];
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) pre[g] += gx4[g];
                const bool valid = !a.len || t < a.len[bb];
                float c = creg[k], hv = hreg[k];
                float4 gates = make_float4(0.f, 0.f, 0.f, 0.f);
                if (valid) {   // padding of a variable-length row holds the state
                    const float ig = sigmoid_f(pre[0]), fg = sigmoid_f(pre[1]);
                    const float gg = tanhf(pre[2]), og = sigmoid_f(pre[3]);
                    c = fg * c + ig * gg;
                    hv = og * tanhf(c);
                    creg[k] = c;
                    hreg[k] = hv;
                    gates = make_float4(ig, fg, gg, og);
                }
                const float hi = tf32_hi(hv);
                hxo[(size_t)bb * 2 * H + u] = hi;
                hxo[(size_t)bb * 2 * H + H + u] = hv - hi;
                if (a.hseq) a.hseq[((size_t)t * B + bb) * ldseq + (size_t)d * H + u] = hv;
                if (a.out) a.out[(size_t)t * a.out_st + (size_t)bb * a.out_sb + (size_t)d * H + u] = valid ? hv : 0.f;
                if (kTrain) {
                    const size_t row = ((size_t)d * T + t) * B + bb;
                    *reinterpret_cast<float4*>(a.act + row * G + 4 * u) = gates;
                    a.cst[row * H + u] = c;
                }
                if (s == T - 1) {
                    a.h_n[((size_t)d * B + bb) * H + u] = hv;
                    a.c_n[((size_t)d * B + bb) * H + u] = c;
                }
            }
            trace_mark(a.trace, tre, s, 7);
            // publish: the exchange writes before the group's TMA reads them
            tc::fence_proxy_async_global();
            tc::named_bar_sync(1, kEpi);
            if (e == 0 && !((int)blockIdx.x == a.skip_block && s == a.skip_step)) red_release_add(ctr, 1u);
            trace_mark(a.trace, tre, s, 8);
        }
    }
    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem, 512);
    }
    cluster_sync();   // no block leaves while another of the cluster may still write into it
}

}  // namespace

TcRec32Plan plan_tc_rec32(int H, int B, int D, int num_sms, size_t smem_max) {
    TcRec32Plan p{};
    // K parts of 128: hi + lo fill the 256 tensor-memory columns beside the
    // accumulator; at least a pair of blocks, at most a portable cluster of 8
    if (H % kMaxKP != 0 || H < 2 * kMaxKP || H > 8 * kMaxKP || B < 1 || D < 1) return p;
    const int C = H / kMaxKP, KP = kMaxKP;
    const int nsl = 4 * H / kRows;
    const int max_groups = num_sms / (C * nsl * D);
    if (max_groups < 1) return p;
    int nbg = std::min(max_groups, std::max(1, (B + 31) / 32));
    int Bg = (B + nbg - 1) / nbg;
    while (((Bg + 31) / 32) * 32 > kMaxN && nbg < max_groups) {
        ++nbg;
        Bg = (B + nbg - 1) / nbg;
    }
    const int N = ((Bg + 31) / 32) * 32;
    if (N > kMaxN || N % (4 * C) != 0) return p;   // own columns in whole quads
    if (nbg > 1 && (nbg - 1) * Bg >= B) return p;
    // alignment, the hi and lo tiles of h, received partial sums, barriers
    const size_t need = 1024 + (size_t)2 * (KP / 32) * N * 128 + (size_t)512 * N + 256;
    if (need > smem_max) return p;
    p.ok = true;
    p.nbg = nbg; p.Bg = Bg; p.N = N; p.nsl = nsl; p.C = C; p.KP = KP;
    p.ctas = C * nsl * D * nbg;
    p.smem = std::min(smem_max, std::max(kMinSmem, need));
    return p;
}

namespace {
typedef CUresult (*EncodeTiledFn32)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
}  // namespace

bool make_map_f32_chunks(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows,
                         int box_chunks) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return false;
    const EncodeTiledFn32 fn = reinterpret_cast<EncodeTiledFn32>(p);
    cuuint64_t dims[3] = {32, (cuuint64_t)rows, (cuuint64_t)(cols / 32)};
    cuuint64_t strides[2] = {(cuuint64_t)(cols * 4), 128};
    cuuint32_t box[3] = {32, (cuuint32_t)box_rows, (cuuint32_t)box_chunks};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_rec32_slot0(const TcRec32Args& a, cudaStream_t s) {
    if (a.T <= 0 || a.B <= 0) return cudaSuccess;
    rec32_slot0_kernel<<<std::min(a.D * a.B, 148 * 16), 256, 0, s>>>(a.h0, a.hx, a.D, a.T, a.B, a.H);
    return cudaGetLastError();
}

cudaError_t launch_tc_rec32(const TcRec32Args& a, cudaStream_t s, int* nlaunch) {
    const TcRec32Plan& p = a.p;
    if (nlaunch) *nlaunch = 0;
    if (!p.ok) return cudaErrorInvalidValue;
    if (a.T <= 0 || a.B <= 0) return cudaSuccess;
    cudaError_t e;
    CUtensorMap tmX;
    const long long rows = (long long)a.D * (a.T + 1) * a.B;
    if (!make_map_f32_chunks(&tmX, a.hx, rows, 2LL * a.H, p.N, p.KP / 32 / kSeg)) return cudaErrorInvalidValue;
    TcRec32Params prm{};
    prm.H = a.H; prm.B = a.B; prm.T = a.T; prm.D = a.D;
    prm.nbg = p.nbg; prm.Bg = p.Bg; prm.N = p.N; prm.nsl = p.nsl; prm.C = p.C; prm.KP = p.KP;
    prm.gx = a.gx; prm.wpk = a.wpk; prm.w[0] = a.w[0]; prm.w[1] = a.w[1]; prm.c0 = a.c0; prm.hx = a.hx;
    prm.hseq = a.hseq; prm.out = a.out; prm.out_st = a.out_st; prm.out_sb = a.out_sb;
    prm.h_n = a.h_n; prm.c_n = a.c_n; prm.act = a.act; prm.cst = a.cst;
    prm.ctr = a.ctr; prm.status = a.status; prm.timeout_ns = a.timeout_ns; prm.len = a.len;
    prm.trace = a.trace;
    prm.skip_block = a.skip_block; prm.skip_step = a.skip_step;
    const auto kern = a.act ? tc_rec32_kernel<true> : tc_rec32_kernel<false>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // the blocks of a launch wait on each other: the device must hold them
    // all at once; directions (independent) run as consecutive launches when
    // it cannot hold all of them together
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess) return e;
    if (p.C * clusters >= p.ctas) {
        e = cudaLaunchKernelEx(&cfg, kern, tmX, prm);
        if (e == cudaSuccess && nlaunch) *nlaunch = 1;
        return e;
    }
    const int per_dir = p.ctas / a.D;
    if (p.C * clusters < per_dir) return cudaErrorCooperativeLaunchTooLarge;
    cfg.gridDim = dim3(per_dir);
    for (int d = 0; d < a.D; ++d) {
        prm.d0 = d;
        e = cudaLaunchKernelEx(&cfg, kern, tmX, prm);
        if (e != cudaSuccess) return e;
    }
    if (nlaunch) *nlaunch = a.D;
    return cudaSuccess;
}

}  // namespace lstm
