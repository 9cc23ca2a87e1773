// Persistent LSTM BPTT recurrence on the sm_100a tensor cores for float32
// problems: the recurrent product W_hh^T da in 3xTF32.
//
// Reverse-mode differentiation of the unrolled cell ("LSTM Forward
// Computation", Loop Unroll; cell: warp_nn "Long Short-Term Memory (LSTM)"
// page, equation block).  For t from the last step of the direction to the
// first, per hidden unit u and batch row b:
//     dh    = dy_t + dh_rec,            dh_rec = (W_hh^T da_{t+1})[u]  (grad_hn at the start)
//     dc    = dc_carry + dh o (1 - tanh^2 c_t)
//     da_i  = dc g i (1 - i),  da_f = dc c_{t-1} f (1 - f),
//     da_g  = dc i (1 - g^2),  da_o = dh tanh(c_t) o (1 - o),   dc_carry = dc f
// and after the first step dh0 = W_hh^T da_0 (+ the pass-through of padding),
// dc0 = dc_carry.  Padding of a variable-length row (t >= len[b]) holds the
// state, so it has no gate gradient and hands dh and dc on unchanged.
//
// The products run as kind::tf32 MMAs on operands split into a tf32 part and
// the float32 remainder (x = hi + lo):
//     W^T da ~= W_hi da_hi + W_hi da_lo + W_lo da_hi,
// the lo*lo term (relative size 2^-22) dropped; sums are float32.
//
// M = 128 hidden units of one slice, N = the batch columns of one group, K =
// 4H gates in the packed order 4u'+q.  A cluster of Cl = H/32 blocks owns
// one slice: block rank k keeps the K part [128k, 128k + 128) of the slice's
// rows of W_hh^T in tensor memory, hi and lo side by side (the A operand),
// multiplies it by the same part of da_{t+1} (hi and lo, from a ring of 4
// exchange slots, in kSeg K segments on a barrier each so the MMAs of the
// first segment run while the next lands) with one issuing warp per product
// into three accumulators, and sends each unit's partial sums to the block
// that owns the unit (128/Cl units per block; asynchronous distributed-
// shared-memory stores completing on the owner's mbarrier).  The owner adds
// the Cl partials, computes the gate gradients of its units, stores them for
// the weight phase and publishes them split hi | lo for the next step; the
// blocks of a (direction, batch group) meet on a counter.  Roles: warp 0 TMA,
// warps 1-3 MMA (whole warps, elect.sync for issue), warps 4-11 partial sums
// and gate gradients.  Every wait is bounded: on a timeout the kernel records
// LSTM_ERR_TIMEOUT.
#include <algorithm>
#include <map>
#include <mutex>
#include <utility>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"
#include "lstm_tc_cluster.cuh"

namespace lstm {
namespace {

constexpr int kRows = 128;                // hidden units per slice (MMA M)
constexpr int kKP = 128;                  // K part (gates) per block: hi + lo fill 256 columns
constexpr int kMaxCl = 16;                // blocks per cluster (H <= 512)
constexpr int kEpi = 256;                 // epilogue threads, warps 4-11
constexpr int kIss = 3;                   // issuing warps, one per product
constexpr int kThreads = 32 * (1 + kIss) + kEpi;
constexpr int kMaxN = 64;                 // batch columns per group
constexpr int kMaxCells = 4;              // gate-gradient cells per epilogue thread
constexpr uint32_t kAcol = 256;           // tensor-memory column of the resident W_hh^T part (hi, then lo)
static_assert(kIss * kMaxN <= (int)kAcol, "the accumulators fit below the resident W_hh^T part");
constexpr int kSlots = 4;                 // ring of gate-gradient exchange slots
constexpr int kSeg = 2;                   // K segments of a step's da tiles, each on its own barrier
constexpr size_t kMinSmem = 120 * 1024;   // two blocks never share an SM (512 TMEM columns each)
constexpr int kCtrStride = 32;
constexpr unsigned kFullMask = 0xffffffffu;

struct TcBwd32Params {
    int H, B, T, D;
    int nbg, Bg, N, nsl, Cl;
    int g0;                    // first (direction, batch group) d * nbg + bg of this launch
    const float* w[2];         // W_hh of each direction as given, [4H][H]: W_hh^T[u][4u'+q] = w[(q*H + u')*H + u]
    const float* act;
    const float* cst;
    const float* c0;
    const float* dy; long long dy_st, dy_sb;
    const float* grad_hn;
    const float* grad_cn;
    float* dG;
    float* dax;                // [D][kSlots][B][8H]: tf32 part | remainder, packed order 4u+q
    float* dh0; float* dc0;
    float* dbpart;
    unsigned* ctr;
    int* status;
    uint64_t timeout_ns;
    const int* len;
    unsigned long long* trace;   // per-step timeline of block 0, or null
    int skip_block, skip_step;   // fault injection (tests of the bounded waits), -1: none
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// sum over src < CL of p[src * stride], in src order: the loads carry no
// guard, so all of them are in flight at once
template <int CL>
__device__ __forceinline__ float sum_sources(const float* p, size_t stride) {
    float v[CL];
#pragma unroll
    for (int src = 0; src < CL; ++src) v[src] = p[src * stride];
    float sum = 0.f;
#pragma unroll
    for (int src = 0; src < CL; ++src) sum += v[src];
    return sum;
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd32_kernel(const __grid_constant__ CUtensorMap tmD, TcBwd32Params a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int N = a.N, Cl = a.Cl, kOwn = kRows / Cl;
    const int nkc = kKP / 32;                             // 32-wide K chunks of the part
    const int tile = N * 128;                             // one chunk of da: N rows x 32 floats
    unsigned char* sBh = smem;                            // [nkc][N][32] hi, 128-byte swizzle
    unsigned char* sBl = smem + nkc * tile;               // the same for lo
    // partial sums received for the own units: [src][N/4 column quads][kOwn] float4
    float4* recv = reinterpret_cast<float4*>(sBl + nkc * tile);
    float* dbred = reinterpret_cast<float*>(recv + (size_t)Cl * (N / 4) * kOwn);   // [kEpi][4]
    uint64_t* full = reinterpret_cast<uint64_t*>(dbred + kEpi * 4);   // [kSeg]
    uint64_t* empty = full + kSeg;
    uint64_t* d_ready = empty + 1;     // the accumulators were read (count kEpi)
    uint64_t* mma_done = d_ready + 1;
    uint64_t* recv_full = mma_done + 1;
    uint64_t* fin = recv_full + 1;     // [kIss] an issuer's own MMAs drained (abort path)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(fin + kIss);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / Cl;
    const int j = cl % a.nsl;
    const int grp = a.g0 + cl / a.nsl;                    // d * nbg + bg
    const int bg = grp % a.nbg, d = grp / a.nbg;
    const int b0 = bg * a.Bg, nB = min(a.Bg, B - b0);
    const int u0 = j * kRows;                             // first unit of the slice
    const int ubeg = u0 + (int)rank * kOwn;               // first own unit
    const int kbeg = (int)rank * kKP;                     // first gate (packed order) of the K part
    const int nblk = a.nsl * Cl;                          // blocks of the (d, bg) group
    unsigned* ctr = a.ctr + (size_t)grp * kCtrStride;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool tr0 = blockIdx.x == 0 && lane == 0 && warp <= 1;              // producer, first issuer
    const bool tre = blockIdx.x == 0 && warp == 1 + kIss && lane == 0;       // an epilogue thread

    if (threadIdx.x == 0) {
        for (int i = 0; i < kSeg; ++i) tc::mbar_init(full + i, 1);
        tc::mbar_init(empty, kIss);    // one commit per issuer
        tc::mbar_init(d_ready, kEpi);
        tc::mbar_init(mma_done, kIss);
        tc::mbar_init(recv_full, 1);   // armed each step with the Cl blocks' bytes
        for (int i = 0; i < kIss; ++i) tc::mbar_init(fin + i, 1);
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
    const int r = q * 32 + lane;             // accumulator row (unit u0 + r) of this thread
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    // Resident W_hh^T rows of the slice, this block's K part: row r on lane
    // r, one tf32 per column; hi at columns kAcol + k, the remainder at
    // kAcol + kKP + k.
    if (warp == 0 && lane == 0) tc::prefetch_tmap(&tmD);
    if (warp > kIss && half == 0) {
        // W_hh^T[u][g] for gate g = 4u' + q is W_hh[q*H + u'][u]: a warp's 32
        // lanes (consecutive u) read 128 contiguous bytes per element
        const float* wcol = a.w[d] + u0 + r;
        for (int c = 0; c < nkc; ++c) {
#pragma unroll
            for (int h16 = 0; h16 < 2; ++h16) {
                uint32_t vh[16], vl[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int g = kbeg + 32 * c + 16 * h16 + i;
                    const float w = wcol[(size_t)((g & 3) * H + (g >> 2)) * H];
                    const float hi = tf32_hi(w);
                    vh[i] = __float_as_uint(hi);
                    vl[i] = __float_as_uint(w - hi);
                }
                tc::tmem_st16(trow + kAcol + (uint32_t)(32 * c + 16 * h16), vh);
                tc::tmem_st16(trow + kAcol + (uint32_t)(kKP + 32 * c + 16 * h16), vl);
            }
        }
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    // every block is resident: a programmatic dependent launched behind this
    // grid (a weight-gradient GEMM of the layer above) may start on the SMs left
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        // ---------------------------------------------------- da producer
        // iteration s (1..T) multiplies the gate gradients of iteration s-1,
        // ring slot s % kSlots; they are complete when every block of the
        // group arrived s times
        int issued = 0;
        for (int s = 1; s <= T; ++s) {
            bool got = true;
            if (lane == 0) got = ctr_wait(ctr, (unsigned)(nblk * s), abort_flag, a.status, a.timeout_ns);
            got = __shfl_sync(kFullMask, got, 0);
            __syncwarp();
            if (!got) break;
            tc::fence_proxy_async_global();
            // the tiles are free once the previous iteration's MMAs completed
            if (s >= 2 &&
                !__all_sync(kFullMask, tc::mbar_wait(empty, (s - 2) & 1, abort_flag, a.status, a.timeout_ns)))
                break;
            trace_mark(a.trace, tr0, s, 0);
            if (tc::elect_one()) {
                const int row0 = (d * kSlots + s % kSlots) * B + b0;
                const int cps = nkc / kSeg;   // chunks per segment
                for (int sg = 0; sg < kSeg; ++sg) {
                    tc::mbar_arrive_expect_tx(full + sg, (uint32_t)(2 * cps * tile));
                    tc::tma_load_3d(sBh + sg * cps * tile, &tmD, 0, row0, kbeg / 32 + sg * cps, full + sg);
                    tc::tma_load_3d(sBl + sg * cps * tile, &tmD, 0, row0, (G + kbeg) / 32 + sg * cps, full + sg);
                }
            }
            __syncwarp();
            ++issued;
        }
        if (*abort_flag && issued > 0)
            for (int sg = 0; sg < kSeg; ++sg) drain_wait(full + sg, (issued - 1) & 1);
    } else if (warp <= kIss) {
        // ------------------------------------------------------------ MMA
        // product pr: A = W_hi (pr < 2) or W_lo, B = da_hi (pr != 1) or da_lo,
        // into the accumulator at column pr * N
        const int pr = warp - 1;
        const uint32_t idesc = tc::instr_desc(2, kRows, N);   // kind::tf32
        const uint32_t acc = tmem + (uint32_t)(pr * N);
        const uint32_t aoff = pr == 2 ? (uint32_t)kKP : 0u;
        const unsigned char* sB = pr == 1 ? sBl : sBh;
        int last = 0;
        for (int s = 1; s <= T; ++s) {
            // the epilogue has read the previous accumulators
            if (!__all_sync(kFullMask, tc::mbar_wait(d_ready, (s - 1) & 1, abort_flag, a.status, a.timeout_ns)))
                break;
            tc::tc_fence_after();
            last = s;   // from here MMAs of iteration s may be in flight (drained on abort)
            bool ok = true;
            const int cps = nkc / kSeg;
            for (int sg = 0; sg < kSeg && ok; ++sg) {
                ok = __all_sync(kFullMask, tc::mbar_wait(full + sg, (s - 1) & 1, abort_flag, a.status, a.timeout_ns));
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
                                            (c | jj) != 0);   // fresh accumulator each iteration
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
        if (*abort_flag && last > 0) {
            // the other issuers may have stopped an iteration earlier: wait
            // for this thread's own MMAs alone
            if (tc::elect_one()) tc::mma_commit(fin + pr);
            __syncwarp();
            drain_wait(fin + pr, 0);
        }
    } else {
        // ------------------------------------------------------- epilogue
        const int e = threadIdx.x - 32 * (1 + kIss);
        // sender: row r's partial sums go to the block that owns unit u0 + r
        const uint32_t dst_rank = (uint32_t)(r / kOwn);
        const int ul_s = r % kOwn;
        const uint32_t recv_dst = map_rank(tc::smem_u32(recv), dst_rank);
        const uint32_t bar_dst = map_rank(tc::smem_u32(recv_full), dst_rank);
        const int colh = half * (N / 2);   // first column of this thread's half
        // owner: cells (unit ubeg + e % kOwn, column (e + kEpi k) / kOwn); a
        // warp's reads of one source cover 128 contiguous bytes
        const int ulo = e % kOwn;
        const int u = ubeg + ulo;
        const int ncell = kOwn * N;
        const size_t ldg = (size_t)D * G;
        const float* rf = reinterpret_cast<const float*>(recv);
        float dcv[kMaxCells], dpass[kMaxCells], dhin[kMaxCells];
        float dbs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kMaxCells; ++k) {
            const int idx = e + kEpi * k;
            const int b = idx / kOwn;
            const bool own = idx < ncell && b < nB;
            const size_t sidx = ((size_t)d * B + b0 + b) * H + u;
            dcv[k] = own && a.grad_cn ? a.grad_cn[sidx] : 0.f;
            dhin[k] = own && a.grad_hn ? a.grad_hn[sidx] : 0.f;
            dpass[k] = 0.f;
        }
        tc::tc_fence_before();
        tc::mbar_arrive(d_ready);   // the accumulators are free for the first MMAs
        bool stop = false;
        for (int s = 0; s <= T && !stop; ++s) {
            const int t = d == 0 ? T - 1 - s : s;   // the step of iteration s < T
            // this step's inputs of the own cells, fetched before the waits
            float4 pact[kMaxCells];
            float pc[kMaxCells], pcp[kMaxCells], pdy[kMaxCells];
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int idx = e + kEpi * k;
                const int b = idx / kOwn;
                pact[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                pc[k] = pcp[k] = pdy[k] = 0.f;
                if (s < T && idx < ncell && b < nB) {
                    const int bb = b0 + b;
                    const size_t row = ((size_t)d * T + t) * B + bb;
                    pact[k] = *reinterpret_cast<const float4*>(a.act + row * G + 4 * u);
                    pc[k] = a.cst[row * H + u];
                    const int tp = d == 0 ? t - 1 : t + 1;
                    if (tp >= 0 && tp < T)
                        pcp[k] = a.cst[(((size_t)d * T + tp) * B + bb) * H + u];
                    else if (a.c0)
                        pcp[k] = a.c0[((size_t)d * B + bb) * H + u];
                    pdy[k] = a.dy[(size_t)t * a.dy_st + (size_t)bb * a.dy_sb + (size_t)d * H + u];
                }
            }
            if (s >= 1) {
                if (e == 0) tc::mbar_arrive_expect_tx(recv_full, (uint32_t)(kRows * N * 4));
                const bool ok = tc::mbar_wait(mma_done, (s - 1) & 1, abort_flag, a.status, a.timeout_ns);
                if (tc::named_bar_or(1, kEpi, !ok)) {
                    stop = true;
                    break;
                }
                tc::tc_fence_after();
                trace_mark(a.trace, tre, s, 4);
                // row r's partial sums over this half's columns: the three
                // products (small cross terms first), then 4-column quads to
                // the owner of the row's unit
                for (int c16 = 0; c16 < N / 32; ++c16) {
                    float v[16], v1[16];
                    const int col = colh + 16 * c16;
                    tc::tmem_ld16(trow + (uint32_t)(N + col), v);       // hi*lo
                    tc::tmem_ld16(trow + (uint32_t)(2 * N + col), v1);  // lo*hi
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += v1[i];
                    tc::tmem_ld16(trow + (uint32_t)col, v1);            // hi*hi
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] += v1[i];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int quad = col / 4 + m;
                        st_async_v4(recv_dst + (uint32_t)((((int)rank * (N / 4) + quad) * kOwn + ul_s) * 16),
                                    v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3], bar_dst);
                    }
                }
                tc::tc_fence_before();
                tc::mbar_arrive(d_ready);   // read: the next MMAs may overwrite the accumulators
                trace_mark(a.trace, tre, s, 5);
                const bool got = mbar_wait_cluster(recv_full, (s - 1) & 1, abort_flag, a.status, a.timeout_ns);
                if (tc::named_bar_or(1, kEpi, !got)) {
                    stop = true;
                    break;
                }
                trace_mark(a.trace, tre, s, 6);
                // the Cl partial sums in a fixed order, plus what padding passed on
#pragma unroll
                for (int k = 0; k < kMaxCells; ++k) {
                    const int idx = e + kEpi * k;
                    if (idx >= ncell) break;
                    const int b = idx / kOwn;
                    const float* p = rf + (((size_t)(b >> 2) * kOwn + ulo) * 4 + (b & 3));
                    const size_t stride = (size_t)(N / 4) * kOwn * 4;
                    const float sum = Cl == 4 ? sum_sources<4>(p, stride)
                                      : Cl == 8 ? sum_sources<8>(p, stride)
                                                : sum_sources<kMaxCl>(p, stride);
                    dhin[k] = sum + dpass[k];
                }
            }
            if (s == T) {   // dh0 = W_hh^T da_0 (+ padding), dc0 = the carry
#pragma unroll
                for (int k = 0; k < kMaxCells; ++k) {
                    const int idx = e + kEpi * k;
                    const int b = idx / kOwn;
                    if (idx >= ncell || b >= nB) continue;
                    const size_t sidx = ((size_t)d * B + b0 + b) * H + u;
                    a.dh0[sidx] = dhin[k];
                    a.dc0[sidx] = dcv[k];
                }
                break;
            }
            // gate gradients of the own cells: dG (standard row order) and the
            // exchange slot of iteration s + 1 (tf32 part | remainder, order 4u+q)
            float* dxo = a.dax + ((size_t)(d * kSlots + (s + 1) % kSlots) * B) * 2 * G + 4 * u;
            float dak[kMaxCells][4];   // this step's gate gradients of the own cells
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int idx = e + kEpi * k;
                const int b = idx / kOwn;
                if (idx >= ncell || b >= nB) continue;
                const int bb = b0 + b;
                float da[4] = {0.f, 0.f, 0.f, 0.f};
                if (a.len && t >= a.len[bb]) {
                    dpass[k] = dhin[k];   // held state: dh and dc pass on, no gate gradient
                } else {
                    dpass[k] = 0.f;
                    const float ig = pact[k].x, fg = pact[k].y, gg = pact[k].z, og = pact[k].w;
                    const float dh = pdy[k] + dhin[k];
                    const float th = tanhf(pc[k]);
                    const float dc = dcv[k] + dh * og * (1.f - th * th);
                    da[0] = dc * gg * ig * (1.f - ig);
                    da[1] = dc * pcp[k] * fg * (1.f - fg);
                    da[2] = dc * ig * (1.f - gg * gg);
                    da[3] = dh * th * og * (1.f - og);
                    dcv[k] = dc * fg;
#pragma unroll
                    for (int g = 0; g < 4; ++g) dbs[g] += da[g];
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) dak[k][g] = da[g];
                float hi[4], lo[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    hi[g] = tf32_hi(da[g]);
                    lo[g] = da[g] - hi[g];
                }
                float* xrow = dxo + (size_t)bb * 2 * G;
                *reinterpret_cast<float4*>(xrow) = make_float4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<float4*>(xrow + G) = make_float4(lo[0], lo[1], lo[2], lo[3]);
            }
            trace_mark(a.trace, tre, s, 7);
            // publish: the exchange writes before the group's TMA reads them
            // (the fence waits for this thread's stores: only the exchange so far)
            tc::fence_proxy_async_global();
            tc::named_bar_sync(1, kEpi);
            if (e == 0 && !((int)blockIdx.x == a.skip_block && s == a.skip_step)) red_release_add(ctr, 1u);
            trace_mark(a.trace, tre, s + 1, 8);
            // then dG, which only the weight phase reads
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int idx = e + kEpi * k;
                const int b = idx / kOwn;
                if (idx >= ncell || b >= nB) continue;
                float* dgp = a.dG + ((size_t)t * B + b0 + b) * ldg + (size_t)d * G + u;
#pragma unroll
                for (int g = 0; g < 4; ++g) dgp[(size_t)g * H] = dak[k][g];
            }
        }
        // bias-gradient partial of the own units over the group's rows, in a
        // fixed order over the threads that share a unit (e = ul + kOwn m)
#pragma unroll
        for (int g = 0; g < 4; ++g) dbred[e * 4 + g] = dbs[g];
        tc::named_bar_sync(1, kEpi);
        if (e < 4 * kOwn) {
            const int g = e / kOwn, ul = e % kOwn;
            float sum = 0.f;
            for (int m = 0; m < kEpi / kOwn; ++m) sum += dbred[(ul + kOwn * m) * 4 + g];
            a.dbpart[((size_t)d * a.nbg + bg) * G + (size_t)g * H + ubeg + ul] = sum;
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

namespace {
// Launch configuration of tc_bwd32_kernel for clusters of Cl blocks.
cudaError_t bwd32_config(int Cl, size_t smem, int ctas, cudaStream_t s, cudaLaunchConfig_t& cfg,
                         cudaLaunchAttribute* attr) {
    cudaError_t e = cudaFuncSetAttribute(tc_bwd32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (Cl > 8) {
        e = cudaFuncSetAttribute(tc_bwd32_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = dim3(ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = Cl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaSuccess;
}

// Clusters of Cl blocks of this kernel the current device holds at once
// (every block of a group waits on the others, so a launch must fit whole).
// Without a device: the counts of a B200 (148 SMs in GPCs of unequal size).
int bwd32_max_clusters(int Cl) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return Cl == 4 ? 33 : Cl == 8 ? 15 : 7;
    }
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(dev, Cl);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    int n = 0;
    if (bwd32_config(Cl, kMinSmem, Cl, nullptr, cfg, attr) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, tc_bwd32_kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    cache[key] = n;
    return n;
}
}  // namespace

TcBwd32Plan plan_tc_bwd32(int H, int B, int D, int num_sms, size_t smem_max) {
    TcBwd32Plan p{};
    // K parts of 128 gates: a cluster of H/32 blocks per 128-unit slice
    if (H % kRows != 0 || B < 1 || D < 1) return p;
    const int Cl = 4 * H / kKP;
    if (Cl != 4 && Cl != 8 && Cl != kMaxCl) return p;
    const int nsl = H / kRows, kOwn = kRows / Cl;
    const int maxc = bwd32_max_clusters(Cl);
    // batch groups of 32 columns when all their clusters fit at once, else of 64
    for (int Nt = 32; Nt <= kMaxN; Nt *= 2) {
        const int nbg = (B + Nt - 1) / Nt;
        const int Bg = (B + nbg - 1) / nbg;
        const int N = ((Bg + 31) / 32) * 32;
        if (N > kMaxN || kOwn * N > kMaxCells * kEpi) continue;
        if (nbg > 1 && (nbg - 1) * Bg >= B) continue;
        if (D * nbg * nsl > maxc || D * nbg * nsl * Cl > num_sms) continue;
        // alignment, da boxes (hi, lo), received partial sums, bias reduction, barriers
        const size_t need = 1024 + (size_t)N * 1024 + (size_t)kRows * N * 4 + (size_t)kEpi * 16 + 256;
        if (need > smem_max) continue;
        p.ok = true;
        p.nbg = nbg; p.Bg = Bg; p.N = N; p.nsl = nsl; p.Cl = Cl;
        p.ctas = Cl * D * nsl * nbg;
        p.smem = std::min(smem_max, std::max(kMinSmem, need));
        p.slots = kSlots;
        return p;
    }
    return p;
}

cudaError_t launch_tc_bwd32(const TcBwd32Args& a, cudaStream_t s, int* nlaunch) {
    if (nlaunch) *nlaunch = 0;
    const TcBwd32Plan& p = a.p;
    if (!p.ok) return cudaErrorInvalidValue;
    if (a.T <= 0 || a.B <= 0) return cudaSuccess;
    CUtensorMap tmD;
    const long long rows = (long long)a.D * kSlots * a.B;
    if (!make_map_f32_chunks(&tmD, a.dax, rows, 8LL * a.H, p.N, kKP / 32 / kSeg)) return cudaErrorInvalidValue;
    TcBwd32Params prm{};
    prm.H = a.H; prm.B = a.B; prm.T = a.T; prm.D = a.D;
    prm.nbg = p.nbg; prm.Bg = p.Bg; prm.N = p.N; prm.nsl = p.nsl; prm.Cl = p.Cl;
    prm.g0 = 0;
    prm.w[0] = a.w[0]; prm.w[1] = a.w[1];
    prm.act = a.act; prm.cst = a.cst; prm.c0 = a.c0;
    prm.dy = a.dy; prm.dy_st = a.dy_st; prm.dy_sb = a.dy_sb;
    prm.grad_hn = a.grad_hn; prm.grad_cn = a.grad_cn;
    prm.dG = a.dG; prm.dax = a.dax;
    prm.dh0 = a.dh0; prm.dc0 = a.dc0; prm.dbpart = a.dbpart;
    prm.ctr = a.ctr; prm.status = a.status; prm.timeout_ns = a.timeout_ns;
    prm.len = a.len;
    prm.trace = a.trace;
    prm.skip_block = a.skip_block; prm.skip_step = a.skip_step;
    cudaLaunchConfig_t cfg;
    cudaLaunchAttribute attr[1];
    cudaError_t e = bwd32_config(p.Cl, p.smem, p.ctas, s, cfg, attr);
    if (e != cudaSuccess) return e;
    // the blocks of a group wait on each other: the launch must fit whole
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, tc_bwd32_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (p.Cl * clusters < p.ctas) return cudaErrorCooperativeLaunchTooLarge;
    e = cudaLaunchKernelEx(&cfg, tc_bwd32_kernel, tmD, prm);
    if (e == cudaSuccess && nlaunch) *nlaunch = 1;
    return e;
}

}  // namespace lstm
