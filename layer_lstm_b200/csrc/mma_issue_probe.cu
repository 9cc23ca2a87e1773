// Issue cost of tcgen05.mma on this device (a measurement tool beside the
// library, not part of it).  One block; one, two or four warps each have one
// elected thread issue a chain of n MMAs (kind::f16, M = 128, K = 16, bf16
// zero operands; B in shared memory, A in shared memory or tensor memory)
// into an accumulator of their own, commit to an mbarrier and wait on it
// (bounded); clock64 is read around the chain, three repetitions after one
// warm-up.  Loop shapes (MODE):
//   0  A in shared memory only (the ss form)
//   1  A in tensor memory only (the ts form)
//   2  both forms compiled in the loop body, a runtime flag picks ss
//   3  both forms compiled in the loop body, a runtime flag picks ts
//   4  two straight loops, n/2 ts MMAs then n/2 ss MMAs (no branch)
//   5  ts only, and before every 4 MMAs a wait on an mbarrier that has
//      already completed plus tcgen05.fence::after_thread_sync, after them
//      a commit to a second mbarrier (a ring of chunk stages, all full)
//   6  ts only, a commit after every 4 MMAs (no wait)
//   7  ts only, the wait and fence before every 4 MMAs (no commit)
//   8  ts only, the wait alone before every 4 MMAs
//   9  ts only, the fence alone before every 4 MMAs
//  10  as 7 with mbarrier.try_wait.relaxed in place of the acquiring wait
//  11  as 7 with mbarrier.test_wait (non-blocking test) in place of try_wait
//  12  the waits of 8 alone, no MMA
//  13  ts only, a volatile shared-memory load before every 4 MMAs
//  14  as 12 with the wait bounded by an iteration count (no clock read);
//      first tries that fail are counted (printed as the last column)
//  15  a %globaltimer read alone in place of each wait of 12
//  16  as 12, each wait on a phase that the thread completes just before
//      (an arrival on a barrier of count 1)
//  17  as 12 with all 32 lanes of the warp executing each wait
//  18  as 12 with try_wait given a suspend-time hint of 0x10 ns
//  19  as 8 (ts, a wait before every 4 MMAs), the whole warp running the
//      loop and waiting, lane 0 issuing the MMAs and the commit
//  20  as 19 with the issuing lane chosen by elect.sync
// Printed as CSV: mode, N, n per warp, warps, cycles of each repetition;
// layer_lstm_b200/mma_probe.py builds it, runs it and turns two chain
// lengths into a marginal cost per MMA.
#include <cstdint>
#include <cstdio>
#include <cuda_runtime.h>

namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// shared-memory matrix descriptor: 128-byte swizzle, 1024-byte stride
// between 8-row groups, sm100 descriptor version
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// instruction descriptor of kind::f16: bf16 A and B, f32 accumulator, both K-major
__host__ __device__ constexpr uint32_t idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ bool try_wait(uint64_t* bar, uint32_t par) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0,1,0,p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(par)
        : "memory");
    return ok;
}
// false after 100 ms; the clock is read only once the first try failed
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t par) {
    if (try_wait(bar, par)) return true;
    const uint64_t t0 = gtimer();
    while (!try_wait(bar, par))
        if (gtimer() - t0 > 100000000ull) return false;
    return true;
}
__device__ __forceinline__ bool try_wait_relaxed(uint64_t* bar, uint32_t par) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.relaxed.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0,1,0,p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(par)
        : "memory");
    return ok;
}
__device__ __forceinline__ bool test_wait(uint64_t* bar, uint32_t par) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0,1,0,p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(par)
        : "memory");
    return ok;
}
// the same bounded wait with either of the two tests above
template <bool kRelaxed>
__device__ __forceinline__ bool wait_bounded_alt(uint64_t* bar, uint32_t par) {
    if (kRelaxed ? try_wait_relaxed(bar, par) : test_wait(bar, par)) return true;
    const uint64_t t0 = gtimer();
    while (!(kRelaxed ? try_wait_relaxed(bar, par) : test_wait(bar, par)))
        if (gtimer() - t0 > 100000000ull) return false;
    return true;
}
// bounded by 2^24 tries; counts a failed first try in *fails
__device__ __forceinline__ bool wait_iter(uint64_t* bar, uint32_t par, int* fails) {
    if (try_wait(bar, par)) return true;
    atomicAdd(fails, 1);
    for (int it = 0; it < (1 << 24); ++it)
        if (try_wait(bar, par)) return true;
    return false;
}
__device__ __forceinline__ bool try_wait_hint(uint64_t* bar, uint32_t par) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0,1,0,p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(par), "r"(0x10u)
        : "memory");
    return ok;
}
__device__ __forceinline__ void mma_ss(uint32_t acc, uint64_t ad, uint64_t bd, uint32_t id, uint32_t accf) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(acc),
        "l"(ad), "l"(bd), "r"(id), "r"(accf)
        : "memory");
}
__device__ __forceinline__ void mma_ts(uint32_t acc, uint32_t at, uint64_t bd, uint32_t id, uint32_t accf) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(acc),
        "r"(at), "l"(bd), "r"(id), "r"(accf)
        : "memory");
}
__device__ __forceinline__ void commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

struct Cfg {
    int N, nmma, nw, flag;
};

constexpr int kSmemA = 128 * 128, kSmemB = 256 * 128;
constexpr uint32_t kAcolT = 480;   // A operand in tensor memory: columns [480, 512)

template <int MODE>
__global__ void __launch_bounds__(128, 1) probe(Cfg c, unsigned long long* out, int* err) {
    extern __shared__ __align__(1024) unsigned char raw[];
    unsigned char* sm = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
    unsigned char* sA = sm;
    unsigned char* sB = sm + kSmemA;
    uint64_t* done = reinterpret_cast<uint64_t*>(sm + kSmemA + kSmemB);   // [4] per issuing warp
    uint64_t* full = done + 4;                                             // completed once, never again
    uint64_t* empty = done + 5;                                            // [4] chunk commits of MODES 5, 6
    uint64_t* fresh = done + 9;                                            // [4] arrive-then-wait of MODE 16
    uint32_t* slot = reinterpret_cast<uint32_t*>(done + 13);
    for (int i = threadIdx.x; i < (kSmemA + kSmemB) / 16; i += 128) reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) {
        for (int i = 0; i < 13; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(done + i)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(full)) : "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(slot)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *slot;
    {   // zero the tensor-memory A operand: each warp its own 32 lanes
        const uint32_t taddr = tmem + kAcolT + ((uint32_t)(warp * 32) << 16);
        for (int col = 0; col < 32; ++col)
            asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr + col), "r"(0u) : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    for (int rep = 0; rep < 4; ++rep) {
        __syncthreads();
        const long long t0 = clock64();
        if (MODE == 17 && warp < c.nw) {
            for (int j = 0; j < c.nmma / 4; ++j)
                if (!wait_bounded(full, 0)) atomicExch(err, 1);
        }
        if ((MODE == 19 || MODE == 20) && warp < c.nw) {
            const uint32_t id = idesc(128, c.N);
            const uint32_t acc = tmem + (uint32_t)(warp * c.N);
            for (int i = 0; i < c.nmma; i += 4) {
                if (!wait_bounded(full, 0)) atomicExch(err, 1);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                uint32_t leader = lane == 0;
                if (MODE == 20)
                    asm volatile("{\n\t.reg .pred p;\n\telect.sync _|p, 0xffffffff;\n\tselp.u32 %0,1,0,p;\n\t}"
                                 : "=r"(leader));
                if (leader)
                    for (int kk = 0; kk < 4; ++kk)
                        mma_ts(acc, tmem + kAcolT + 8 * kk, desc_sw128(smem_u32(sB) + 32 * kk), id, (i | kk) > 0);
                __syncwarp();
            }
            if (lane == 0) commit(done + warp);
            __syncwarp();
            if (!wait_bounded(done + warp, rep & 1)) atomicExch(err, 1);
        }
        if (MODE != 19 && MODE != 20 && warp < c.nw && lane == 0) {
            const uint32_t id = idesc(128, c.N);
            const uint32_t acc = tmem + (uint32_t)(warp * c.N);   // columns [N w, N w + N)
            uint32_t fresh_phase = (uint32_t)(rep * (c.nmma / 4));   // phases completed on fresh[warp] so far
            if (MODE == 4) {
                const int half = c.nmma / 2;
                for (int i = 0; i < half; ++i) {
                    const int kk = i & 3;
                    mma_ts(acc, tmem + kAcolT + 8 * kk, desc_sw128(smem_u32(sB) + 32 * kk), id, i > 0);
                }
                for (int i = half; i < c.nmma; ++i) {
                    const int kk = i & 3;
                    mma_ss(acc, desc_sw128(smem_u32(sA) + 32 * kk), desc_sw128(smem_u32(sB) + 32 * kk), id, 1);
                }
            } else if (MODE >= 5) {
                for (int i = 0; i < c.nmma; ++i) {
                    const int kk = i & 3;
                    if (kk == 0) {
                        bool ok = true;
                        if (MODE == 5 || MODE == 7 || MODE == 8 || MODE == 12) ok = wait_bounded(full, 0);
                        if (MODE == 10) ok = wait_bounded_alt<true>(full, 0);
                        if (MODE == 11) ok = wait_bounded_alt<false>(full, 0);
                        if (MODE == 14) ok = wait_iter(full, 0, err + 1);
                        if (MODE == 15 && gtimer() == 0ull) ok = false;
                        if (MODE == 18) {
                            ok = false;
                            for (int it = 0; it < (1 << 24) && !ok; ++it) ok = try_wait_hint(full, 0);
                        }
                        if (MODE == 16) {
                            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(fresh + warp)) : "memory");
                            ok = wait_bounded(fresh + warp, fresh_phase & 1);
                            ++fresh_phase;
                        }
                        if (!ok) atomicExch(err, 1);
                        if (MODE != 6 && MODE != 8 && MODE < 12) asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    }
                    if (MODE == 13 && kk == 0) {
                        uint32_t v;
                        asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(slot)) : "memory");
                        if (v == 0xFFFFFFFFu) atomicExch(err, 2);
                    }
                    if (MODE < 12 || MODE == 13) mma_ts(acc, tmem + kAcolT + 8 * kk, desc_sw128(smem_u32(sB) + 32 * kk), id, i > 0);
                    if ((MODE == 5 || MODE == 6) && kk == 3) commit(empty + warp);
                }
            } else {
                for (int i = 0; i < c.nmma; ++i) {
                    const int kk = i & 3;
                    const bool ts = MODE == 1 || (MODE >= 2 && c.flag);
                    if (MODE == 0 || (MODE >= 2 && !ts))
                        mma_ss(acc, desc_sw128(smem_u32(sA) + 32 * kk), desc_sw128(smem_u32(sB) + 32 * kk), id, i > 0);
                    else
                        mma_ts(acc, tmem + kAcolT + 8 * kk, desc_sw128(smem_u32(sB) + 32 * kk), id, i > 0);
                }
            }
            commit(done + warp);
            if (!wait_bounded(done + warp, rep & 1)) atomicExch(err, 1);
        }
        __syncthreads();
        const long long t1 = clock64();
        if (threadIdx.x == 0) out[rep] = (unsigned long long)(t1 - t0);
    }
    if ((MODE == 5 || MODE == 6) && warp < c.nw && lane == 0) {
        // the chunk commits of the last repetition land with its final commit;
        // wait for their count (4 n / 4 arrivals, i.e. n / 4 phase flips)
        const int flips = 4 * (c.nmma / 4);
        if (!wait_bounded(empty + warp, (flips - 1) & 1)) atomicExch(err, 1);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

template <int MODE>
bool run(Cfg c, unsigned long long* d_out, int* d_err, int smem) {
    if (cudaFuncSetAttribute(probe<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return false;
    probe<MODE><<<1, 128, smem>>>(c, d_out, d_err);
    return cudaDeviceSynchronize() == cudaSuccess;
}

}  // namespace

int main() {
    unsigned long long* d_out;
    int* d_err;
    if (cudaMalloc(&d_out, 4 * sizeof(unsigned long long)) != cudaSuccess || cudaMalloc(&d_err, 2 * sizeof(int)) != cudaSuccess)
        return 2;
    cudaMemset(d_err, 0, 2 * sizeof(int));
    const int smem = kSmemA + kSmemB + 1024 + 128;
    printf("mode,N,nmma_per_warp,warps,cyc_rep1,cyc_rep2,cyc_rep3,first_try_fails\n");
    for (int mode = 0; mode < 21; ++mode)
        for (int N : {32, 128, 256})
            for (int nw : {1, 2, 4})
                for (int n : {16, 64}) {
                    if (N * nw > (int)kAcolT) continue;   // accumulators stay clear of the A operand
                    const Cfg c{N, n, nw, mode == 3 ? 1 : 0};
                    bool ok = false;
                    switch (mode) {
                        case 0: ok = run<0>(c, d_out, d_err, smem); break;
                        case 1: ok = run<1>(c, d_out, d_err, smem); break;
                        case 2: case 3: ok = run<2>(c, d_out, d_err, smem); break;
                        case 4: ok = run<4>(c, d_out, d_err, smem); break;
                        case 5: ok = run<5>(c, d_out, d_err, smem); break;
                        case 6: ok = run<6>(c, d_out, d_err, smem); break;
                        case 7: ok = run<7>(c, d_out, d_err, smem); break;
                        case 8: ok = run<8>(c, d_out, d_err, smem); break;
                        case 9: ok = run<9>(c, d_out, d_err, smem); break;
                        case 10: ok = run<10>(c, d_out, d_err, smem); break;
                        case 11: ok = run<11>(c, d_out, d_err, smem); break;
                        case 12: ok = run<12>(c, d_out, d_err, smem); break;
                        case 13: ok = run<13>(c, d_out, d_err, smem); break;
                        case 14: ok = run<14>(c, d_out, d_err, smem); break;
                        case 15: ok = run<15>(c, d_out, d_err, smem); break;
                        case 16: ok = run<16>(c, d_out, d_err, smem); break;
                        case 17: ok = run<17>(c, d_out, d_err, smem); break;
                        case 18: ok = run<18>(c, d_out, d_err, smem); break;
                        case 19: ok = run<19>(c, d_out, d_err, smem); break;
                        default: ok = run<20>(c, d_out, d_err, smem); break;
                    }
                    if (!ok) {
                        printf("error\n");
                        return 1;
                    }
                    unsigned long long h[4];
                    int fails = 0;
                    cudaMemcpy(h, d_out, sizeof(h), cudaMemcpyDeviceToHost);
                    cudaMemcpy(&fails, d_err + 1, sizeof(int), cudaMemcpyDeviceToHost);
                    cudaMemset(d_err + 1, 0, sizeof(int));
                    printf("%d,%d,%d,%d,%llu,%llu,%llu,%d\n", mode, N, n, nw, h[1], h[2], h[3], fails);
                }
    int herr = 0;
    cudaMemcpy(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost);
    printf("err=%d\n", herr);
    return herr;
}
