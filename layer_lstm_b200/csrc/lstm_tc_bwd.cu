// Persistent LSTM BPTT recurrence on the sm_100a tensor cores (bf16 W_hh).
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
// The products dh_rec = W_hh^T da are the tensor-core part: M = 128 hidden
// units of one slice, N = the batch columns of one group, K = 4H gates in the
// packed order 4u'+q.  A cluster of 8 blocks owns one slice: block rank k
// keeps the K part [k*H/2, (k+1)*H/2) of its 128 rows of W_hh^T resident in
// tensor memory (the A operand of tcgen05.mma), multiplies it by the same
// part of da_{t+1} (TMA, one 3-D box per step) and sends each unit's partial
// sums to the block that owns the unit (16 units per block; asynchronous
// distributed-shared-memory stores completing on the owner's mbarrier).  The
// owner adds the 8 partials, computes the gate gradients of its 16 units,
// stores them (for the weight phase, float32 or bf16) and publishes them in bf16 for
// the next step; the blocks of a (direction, batch group) meet on a counter,
// as in the tensor-core forward.  Roles: warp 0 TMA, warp 1 MMA (both whole
// warps, elect.sync for issue), warps 2-9 partial sums and gate gradients.
// Every wait is bounded: on a timeout the kernel records LSTM_ERR_TIMEOUT.
#include <algorithm>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"
#include "lstm_tc_cluster.cuh"

namespace lstm {
namespace {

constexpr int kRows = 128;                // hidden units per slice (MMA M)
constexpr int kCl = 8;                    // blocks per cluster: K parts
constexpr int kOwn = kRows / kCl;         // units owned by each block of a cluster
constexpr int kEpi = 256;                 // epilogue threads, warps 2-9
constexpr int kThreads = 64 + kEpi;
constexpr int kMaxN = 64;                 // batch columns per group (4 cells per epilogue thread)
constexpr int kMaxCells = kOwn * kMaxN / kEpi;   // gate-gradient cells per epilogue thread
constexpr uint32_t kAcol = 256;           // tensor-memory column of the resident W_hh^T part
constexpr int kMaxChunks = 8;             // 8 x 32 columns of W_hh^T (64 gates each)
constexpr size_t kMinSmem = 120 * 1024;   // two blocks never share an SM (512 TMEM columns each)
constexpr int kCtrStride = 32;
constexpr unsigned kFullMask = 0xffffffffu;

struct TcBwdParams {
    int H, B, T, D;
    int nbg, Bg, N, nsl, nch;
    int d0;                    // first direction of this launch
    const bf16* wT;
    const float* act;
    const float* cst;
    const float* c0;
    const float* dy; long long dy_st, dy_sb;
    const float* grad_hn;
    const float* grad_cn;
    void* dG;
    int dG_bf16;
    bf16* dax;
    float* dh0; float* dc0;
    float* dbpart;
    unsigned* ctr;
    int* status;
    uint64_t timeout_ns;
    const int* len;
};

// out[d][u][4u'+q] = W[d][q*H + u'][u]: a 32 x 32 tile transpose per gate q
// (bf16 for this kernel, float32 for the 3xTF32 one).
template <typename E>
__global__ void pack_wT_kernel(PackWtArgs a) {
    __shared__ E tile[32][34];
    const int H = a.H;
    const int u0 = blockIdx.x * 32, v0 = blockIdx.y * 32;   // u: column of W (row of out), v = u'
    const int q = blockIdx.z % 4, d = blockIdx.z / 4;
    const E* w = static_cast<const E*>(a.w[d]);
    E* out = static_cast<E*>(a.out) + (size_t)d * H * 4 * H;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8 threads
    for (int i = ty; i < 32; i += 8) {
        const int v = v0 + i, u = u0 + tx;
        tile[i][tx] = (v < H && u < H) ? w[((size_t)q * H + v) * H + u] : E(0.f);
    }
    __syncthreads();
    for (int i = ty; i < 32; i += 8) {
        const int u = u0 + i, v = v0 + tx;
        if (u < H && v < H) out[(size_t)u * 4 * H + 4 * v + q] = tile[tx][i];
    }
}

__global__ void __launch_bounds__(kThreads, 1)
    tc_bwd_kernel(const __grid_constant__ CUtensorMap tmD, TcBwdParams a) {
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int N = a.N, nch = a.nch;
    const int bstage = nch * N * 128;                    // this block's K part of da, one box
    unsigned char* sB = smem;
    // partial sums received from the 8 blocks of the cluster for the own
    // units: [source][N/4 column quads][kOwn units] float4
    float4* recv = reinterpret_cast<float4*>(sB + bstage);
    float* dbred = reinterpret_cast<float*>(recv + (size_t)kCl * (N / 4) * kOwn);   // [kEpi][4]
    uint64_t* full = reinterpret_cast<uint64_t*>(dbred + kEpi * 4);
    uint64_t* empty = full + 1;
    uint64_t* d_ready = empty + 1;     // the accumulator was read (count kEpi)
    uint64_t* mma_done = d_ready + 1;
    uint64_t* recv_full = mma_done + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_full + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const uint32_t rank = cluster_rank();
    const int cl = blockIdx.x / kCl;
    const int j = cl % a.nsl;
    const int bg = (cl / a.nsl) % a.nbg;
    const int d = a.d0 + cl / (a.nsl * a.nbg);
    const int b0 = bg * a.Bg, nB = min(a.Bg, B - b0);
    const int u0 = j * kRows;                            // first unit of the slice
    const int ubeg = u0 + (int)rank * kOwn;              // first own unit
    const int cbeg = (int)rank * nch;                    // first 64-gate chunk of the K part
    const int nblk = a.nsl * kCl;                        // blocks of the (d, bg) group
    unsigned* ctr = a.ctr + (size_t)(d * a.nbg + bg) * kCtrStride;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tc::mbar_init(full, 1);
        tc::mbar_init(empty, 1);
        tc::mbar_init(d_ready, kEpi);
        tc::mbar_init(mma_done, 1);
        tc::mbar_init(recv_full, 1);   // armed each step with the 8 blocks' bytes
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
    const int half = (warp - 2) >> 2;        // 0 or 1 for epilogue warps
    const int r = q * 32 + lane;             // accumulator row (unit u0 + r) of this thread
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    // Resident W_hh^T rows of the slice, this block's K part: row r on lane
    // r, two bf16 per column, chunk c at columns kAcol + 32c.
    if (warp == 0 && lane == 0) tc::prefetch_tmap(&tmD);
    if (warp >= 2 && half == 0) {
        const bf16* wrow = a.wT + ((size_t)d * H + u0 + r) * G;
        for (int c = 0; c < nch; ++c) {
            const uint4* src = reinterpret_cast<const uint4*>(wrow + 64 * (cbeg + c));
            uint32_t v0[16], v1[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 x = src[i];
                v0[4 * i] = x.x; v0[4 * i + 1] = x.y; v0[4 * i + 2] = x.z; v0[4 * i + 3] = x.w;
                const uint4 y = src[4 + i];
                v1[4 * i] = y.x; v1[4 * i + 1] = y.y; v1[4 * i + 2] = y.z; v1[4 * i + 3] = y.w;
            }
            tc::tmem_st16(trow + kAcol + (uint32_t)c * 32, v0);
            tc::tmem_st16(trow + kAcol + (uint32_t)c * 32 + 16, v1);
        }
        tc::tmem_st_wait();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();

    if (warp == 0) {
        // ---------------------------------------------------- da producer
        // iteration s (1..T) multiplies the gate gradients of iteration s-1,
        // exchange slot s; they are complete when every block of the group
        // arrived s times
        int issued = 0;
        for (int s = 1; s <= T; ++s) {
            bool got = true;
            if (lane == 0) got = ctr_wait(ctr, (unsigned)(nblk * s), abort_flag, a.status, a.timeout_ns);
            got = __shfl_sync(kFullMask, got, 0);
            __syncwarp();
            if (!got) break;
            tc::fence_proxy_async_global();
            // the stage is free once the previous iteration's MMAs completed
            if (s >= 2 &&
                !__all_sync(kFullMask, tc::mbar_wait(empty, (s - 2) & 1, abort_flag, a.status, a.timeout_ns)))
                break;
            if (tc::elect_one()) {
                tc::mbar_arrive_expect_tx(full, (uint32_t)bstage);
                tc::tma_load_3d(sB, &tmD, 0, (d * (T + 1) + s) * B + b0, cbeg, full);
            }
            __syncwarp();
            ++issued;
        }
        if (*abort_flag && issued > 0) drain_wait(full, (issued - 1) & 1);
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        const uint32_t idesc = tc::instr_desc(1, kRows, N);
        int last = 0;
        for (int s = 1; s <= T; ++s) {
            // the epilogue has read the previous accumulator
            if (!__all_sync(kFullMask, tc::mbar_wait(d_ready, (s - 1) & 1, abort_flag, a.status, a.timeout_ns)))
                break;
            tc::tc_fence_after();
            if (!__all_sync(kFullMask, tc::mbar_wait(full, (s - 1) & 1, abort_flag, a.status, a.timeout_ns)))
                break;
            tc::tc_fence_after();
            if (tc::elect_one()) {
                for (int c = 0; c < nch; ++c) {
                    const uint32_t b_base = tc::smem_u32(sB + c * N * 128);
                    const uint32_t at = tmem + kAcol + (uint32_t)c * 32;
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj)
                        tc::mma_bf16_ts(tmem, at + 8 * jj, tc::smem_desc_sw128(b_base + 32 * jj), idesc,
                                        (c | jj) != 0);
                }
                tc::mma_commit(empty);
                tc::mma_commit(mma_done);
            }
            __syncwarp();
            last = s;
        }
        if (*abort_flag && last > 0) drain_wait(empty, (last - 1) & 1);
    } else {
        // ------------------------------------------------------- epilogue
        const int e = threadIdx.x - 64;
        // sender: row r's partial sums go to the block that owns unit u0 + r
        const uint32_t dst_rank = (uint32_t)(r / kOwn);
        const int ul_s = r % kOwn;
        const uint32_t recv_dst = map_rank(tc::smem_u32(recv), dst_rank);
        const uint32_t bar_dst = map_rank(tc::smem_u32(recv_full), dst_rank);
        const int colh = half * (N / 2);   // first column of this thread's half
        // owner: cells (unit ubeg + ulo, column e / kOwn + 16k), k < N / 16
        const int ulo = e % kOwn;
        const int u = ubeg + ulo;
        const int ncell = N / 16;
        const size_t ldg = (size_t)D * G;
        float dcv[kMaxCells], dpass[kMaxCells], dhin[kMaxCells];
        float dbs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < kMaxCells; ++k) {
            const int b = e / kOwn + 16 * k;
            const bool own = k < ncell && b < nB;
            const size_t sidx = ((size_t)d * B + b0 + b) * H + u;
            dcv[k] = own && a.grad_cn ? a.grad_cn[sidx] : 0.f;
            dhin[k] = own && a.grad_hn ? a.grad_hn[sidx] : 0.f;
            dpass[k] = 0.f;
        }
        tc::tc_fence_before();
        tc::mbar_arrive(d_ready);   // the accumulator is free for the first MMAs
        bool stop = false;
        for (int s = 0; s <= T && !stop; ++s) {
            const int t = d == 0 ? T - 1 - s : s;   // the step of iteration s < T
            // this step's inputs of the own cells, fetched before the waits
            float4 pact[kMaxCells];
            float pc[kMaxCells], pcp[kMaxCells], pdy[kMaxCells];
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int b = e / kOwn + 16 * k;
                pact[k] = make_float4(0.f, 0.f, 0.f, 0.f);
                pc[k] = pcp[k] = pdy[k] = 0.f;
                if (s < T && k < ncell && b < nB) {
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
                if (e == 0) tc::mbar_arrive_expect_tx(recv_full, (uint32_t)(kCl * kOwn * N * 4));
                const bool ok = tc::mbar_wait(mma_done, (s - 1) & 1, abort_flag, a.status, a.timeout_ns);
                if (tc::named_bar_or(1, kEpi, !ok)) {
                    stop = true;
                    break;
                }
                tc::tc_fence_after();
                // this row's partial sums over the thread's half of the columns
                for (int c16 = 0; c16 < N / 32; ++c16) {
                    float v[16];
                    const int col = colh + 16 * c16;
                    tc::tmem_ld16(trow + (uint32_t)col, v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const int quad = col / 4 + m;
                        st_async_v4(recv_dst + (uint32_t)((((int)rank * (N / 4) + quad) * kOwn + ul_s) * 16),
                                    v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3], bar_dst);
                    }
                }
                tc::tc_fence_before();
                tc::mbar_arrive(d_ready);   // read: the next MMAs may overwrite the accumulator
                const bool got = mbar_wait_cluster(recv_full, (s - 1) & 1, abort_flag, a.status, a.timeout_ns);
                if (tc::named_bar_or(1, kEpi, !got)) {
                    stop = true;
                    break;
                }
                // the 8 partial sums in a fixed order, plus what padding passed on
#pragma unroll
                for (int k = 0; k < kMaxCells; ++k) {
                    if (k >= ncell) break;
                    const int b = e / kOwn + 16 * k;
                    float sum = 0.f;
                    for (int src = 0; src < kCl; ++src) {
                        const float4 p4 = recv[((size_t)src * (N / 4) + b / 4) * kOwn + ulo];
                        const int w = b & 3;
                        sum += w == 0 ? p4.x : w == 1 ? p4.y : w == 2 ? p4.z : p4.w;
                    }
                    dhin[k] = sum + dpass[k];
                }
            }
            if (s == T) {   // dh0 = W_hh^T da_0 (+ padding), dc0 = the carry
#pragma unroll
                for (int k = 0; k < kMaxCells; ++k) {
                    const int b = e / kOwn + 16 * k;
                    if (k >= ncell || b >= nB) continue;
                    const size_t sidx = ((size_t)d * B + b0 + b) * H + u;
                    a.dh0[sidx] = dhin[k];
                    a.dc0[sidx] = dcv[k];
                }
                break;
            }
            // gate gradients of the own cells: dG (float32, standard row
            // order) and the exchange slot s + 1 (bf16, order 4u+q)
            bf16* dxo = a.dax + ((size_t)(d * (T + 1) + s + 1) * B) * G + 4 * u;
#pragma unroll
            for (int k = 0; k < kMaxCells; ++k) {
                const int b = e / kOwn + 16 * k;
                if (k >= ncell || b >= nB) continue;
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
                const size_t gi = ((size_t)t * B + bb) * ldg + (size_t)d * G + u;
                if (a.dG_bf16) {
                    bf16* dgp = static_cast<bf16*>(a.dG) + gi;
#pragma unroll
                    for (int g = 0; g < 4; ++g) dgp[(size_t)g * H] = __float2bfloat16_rn(da[g]);
                } else {
                    float* dgp = static_cast<float*>(a.dG) + gi;
#pragma unroll
                    for (int g = 0; g < 4; ++g) dgp[(size_t)g * H] = da[g];
                }
                const __nv_bfloat162 p01 = __floats2bfloat162_rn(da[0], da[1]);
                const __nv_bfloat162 p23 = __floats2bfloat162_rn(da[2], da[3]);
                uint2 pk;
                pk.x = *reinterpret_cast<const uint32_t*>(&p01);
                pk.y = *reinterpret_cast<const uint32_t*>(&p23);
                *reinterpret_cast<uint2*>(dxo + (size_t)bb * G) = pk;
            }
            // publish: the exchange writes before the group's TMA reads them
            tc::fence_proxy_async_global();
            tc::named_bar_sync(1, kEpi);
            if (e == 0) red_release_add(ctr, 1u);
        }
        // bias-gradient partial of the own units over the group's rows, in a
        // fixed order over the threads that share a unit
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

TcBwdPlan plan_tc_bwd(int H, int B, int D, int num_sms, size_t smem_max) {
    TcBwdPlan p{};
    // 128-unit slices; a K part of H/2 gates is at most 8 chunks of 64
    if (H % kRows != 0 || H > kRows * kMaxChunks || B < 1 || D < 1) return p;
    const int nsl = H / kRows;
    const int nch = (4 * H / kCl) / 64;
    const int max_groups = num_sms / (kCl * D * nsl);
    if (max_groups < 1) return p;
    int nbg = std::min(max_groups, std::max(1, (B + 31) / 32));
    int Bg = (B + nbg - 1) / nbg;
    while (((Bg + 31) / 32) * 32 > kMaxN && nbg < max_groups) {
        ++nbg;
        Bg = (B + nbg - 1) / nbg;
    }
    const int N = ((Bg + 31) / 32) * 32;
    if (N > kMaxN) return p;
    if (nbg > 1 && (nbg - 1) * Bg >= B) return p;
    // alignment, da box, received partial sums, bias reduction, barriers
    const size_t need = 1024 + (size_t)nch * N * 128 + (size_t)kCl * kOwn * N * 4 + (size_t)kEpi * 16 + 256;
    if (need > smem_max) return p;
    p.ok = true;
    p.nbg = nbg; p.Bg = Bg; p.N = N; p.nsl = nsl; p.nch = nch;
    p.ctas = kCl * D * nsl * nbg;
    p.smem = std::min(smem_max, std::max(kMinSmem, need));
    return p;
}

cudaError_t launch_pack_wT(const PackWtArgs& a, cudaStream_t s) {
    if (a.H <= 0 || a.D <= 0) return cudaSuccess;
    const dim3 grid((a.H + 31) / 32, (a.H + 31) / 32, 4 * a.D);
    if (a.dt == DType::F32)
        pack_wT_kernel<float><<<grid, 256, 0, s>>>(a);
    else
        pack_wT_kernel<bf16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_tc_bwd(const TcBwdArgs& a, cudaStream_t s, int* nlaunch) {
    if (nlaunch) *nlaunch = 1;
    const TcBwdPlan& p = a.p;
    if (!p.ok) return cudaErrorInvalidValue;
    if (a.T <= 0 || a.B <= 0) return cudaSuccess;
    CUtensorMap tmD;
    const long long rows = (long long)a.D * (a.T + 1) * a.B;
    if (!make_map_bf16_chunks(&tmD, a.dax, rows, 4LL * a.H, p.N, p.nch)) return cudaErrorInvalidValue;
    TcBwdParams prm{};
    prm.H = a.H; prm.B = a.B; prm.T = a.T; prm.D = a.D;
    prm.nbg = p.nbg; prm.Bg = p.Bg; prm.N = p.N; prm.nsl = p.nsl; prm.nch = p.nch;
    prm.wT = static_cast<const bf16*>(a.wT);
    prm.act = a.act; prm.cst = a.cst; prm.c0 = a.c0;
    prm.dy = a.dy; prm.dy_st = a.dy_st; prm.dy_sb = a.dy_sb;
    prm.grad_hn = a.grad_hn; prm.grad_cn = a.grad_cn;
    prm.dG = a.dG; prm.dG_bf16 = a.dG_bf16; prm.dax = static_cast<bf16*>(a.dax);
    prm.dh0 = a.dh0; prm.dc0 = a.dc0; prm.dbpart = a.dbpart;
    prm.ctr = a.ctr; prm.status = a.status; prm.timeout_ns = a.timeout_ns;
    prm.len = a.len;
    cudaError_t e = cudaFuncSetAttribute(tc_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(p.ctas);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCl;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // Every block waits on the others of its (direction, group), so the
    // blocks of a launch must be resident at once.  Clusters of 8 fill a GPC
    // unevenly: when the device cannot hold all directions together, the
    // directions (independent of each other) run as consecutive launches.
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, tc_bwd_kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (kCl * clusters >= p.ctas) return cudaLaunchKernelEx(&cfg, tc_bwd_kernel, tmD, prm);
    const int per_dir = p.ctas / a.D;
    if (kCl * clusters < per_dir) return cudaErrorCooperativeLaunchTooLarge;
    cfg.gridDim = dim3(per_dir);
    if (nlaunch) *nlaunch = a.D;
    for (int d = 0; d < a.D; ++d) {
        prm.d0 = d;
        e = cudaLaunchKernelEx(&cfg, tc_bwd_kernel, tmD, prm);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace lstm
