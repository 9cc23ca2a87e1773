// Issue cost of tcgen05.mma on this device (measurement tool, not part of
// the library): one thread of one block (or of every block of a 148-block
// grid) issues a chain of n MMAs (kind::f16, K = 16) with zero operands
// resident in shared memory (A optionally in tensor memory) into one or
// four accumulators, commits, waits on the mbarrier (bounded), and reads
// clock64 around the chain; four repetitions per configuration.  Printed as
// CSV: grid, M, N, n, accumulators, A in tensor memory, per-chunk commits,
// cycles of each repetition.  The design of the tensor-core recurrence rests
// on the result: the chain costs the same per instruction for every N from
// 16 to 256 and M of 64 or 128, so a step's time follows its instruction
// count.  Built and run by layer_lstm_b200/mma_probe.py.
#include <cstdio>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <vector>

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ uint64_t gtimer() { uint64_t t; asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t)); return t; }
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__host__ __device__ constexpr uint32_t idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ bool try_wait(uint64_t* bar, uint32_t par) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0,1,0,p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(par) : "memory");
    return ok;
}
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t par) {
    uint64_t t0 = gtimer();
    while (!try_wait(bar, par)) if (gtimer() - t0 > 100000000ull) return false;
    return true;
}

struct Cfg { int M, N, nmma, nacc, a_tmem, chunk_wait; };

__global__ void __launch_bounds__(128, 1) probe(Cfg c, unsigned long long* out, int* err) {
    extern __shared__ __align__(1024) unsigned char raw[];
    unsigned char* sm = raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
    unsigned char* sA = sm;              // 128 rows x 128 B
    unsigned char* sB = sm + 16384;      // 256 rows x 128 B
    uint64_t* bar = reinterpret_cast<uint64_t*>(sm + 16384 + 32768);
    uint64_t* bar2 = bar + 1;
    uint32_t* slot = reinterpret_cast<uint32_t*>(bar + 2);
    for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += 128) reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar)) : "memory");
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_u32(bar2)) : "memory");
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    const int warp = threadIdx.x >> 5;
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(slot)) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *slot;
    // zero A region in tmem cols 256..287 (all 4 warps, own lane quarter)
    {
        uint32_t z = 0;
        uint32_t taddr = tmem + 256 + ((uint32_t)(warp * 32) << 16);
        for (int cidx = 0; cidx < 32; cidx += 1)
            asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr + cidx), "r"(z) : "memory");
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    if (threadIdx.x == 0) {
        const uint32_t id = idesc(c.M, c.N);
        uint32_t par = 0;
        for (int rep = 0; rep < 4; ++rep) {
            long long t0 = clock64();
            for (int i = 0; i < c.nmma; ++i) {
                const uint32_t acc = (uint32_t)((i % c.nacc) * c.N);
                const uint32_t accf = i >= c.nacc ? 1u : 0u;
                const int kk = i & 3;
                const uint64_t bd = desc_sw128(smem_u32(sB) + 32 * kk);
                if (c.a_tmem) {
                    const uint32_t at = tmem + 256 + 8 * kk;
                    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
                                 ::"r"(tmem + acc), "r"(at), "l"(bd), "r"(id), "r"(accf) : "memory");
                } else {
                    const uint64_t ad = desc_sw128(smem_u32(sA) + 32 * kk);
                    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                                 ::"r"(tmem + acc), "l"(ad), "l"(bd), "r"(id), "r"(accf) : "memory");
                }
                if (c.chunk_wait && (i & 3) == 3) {
                    // commit per 4 MMAs (like a per-chunk empty barrier), no wait
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar2)) : "memory");
                }
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
            if (!wait_bounded(bar, par)) { atomicExch(err, 1); wait_bounded(bar, par); }
            par ^= 1;
            long long t1 = clock64();
            if (blockIdx.x == 0) out[rep] = (unsigned long long)(t1 - t0);
        }
        // drain bar2 arrivals are fire-and-forget (count 1 barrier just flips); nothing to wait
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

int main() {
    unsigned long long* d_out; int* d_err;
    cudaMalloc(&d_out, 64 * sizeof(unsigned long long));
    cudaMalloc(&d_err, sizeof(int));
    cudaMemset(d_err, 0, sizeof(int));
    const int smem = 16384 + 32768 + 1024 + 64;
    cudaFuncSetAttribute(probe, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    std::vector<Cfg> cfgs;
    for (int a = 0; a < 2; ++a)
        for (int N : {16, 32, 64, 128, 256})
            for (int n : {1, 4, 16, 64})
                for (int nacc : {1, 4}) {
                    if (a && N * nacc > 256) continue;
                    if (!a && N * nacc > 512) continue;
                    cfgs.push_back({128, N, n, nacc, a, 0});
                }
    for (int N : {32, 64, 128, 256})
        for (int n : {1, 16, 64}) cfgs.push_back({64, N, n, 1, 0, 0});
    for (int N : {32, 256}) cfgs.push_back({128, N, 64, 1, 1, 1});
    int grids[2] = {1, 148};
    printf("grid,M,N,nmma,nacc,a_tmem,chunk_commit,cyc_rep0,cyc_rep1,cyc_rep2,cyc_rep3\n");
    for (int g = 0; g < 2; ++g) {
        for (const Cfg& c : cfgs) {
            if (g == 1 && !(c.nmma == 64 && c.nacc == 1)) continue;
            probe<<<grids[g], 128, smem>>>(c, d_out, d_err);
            cudaError_t e = cudaDeviceSynchronize();
            if (e != cudaSuccess) { printf("error %s\n", cudaGetErrorString(e)); return 1; }
            unsigned long long h[4];
            cudaMemcpy(h, d_out, sizeof(h), cudaMemcpyDeviceToHost);
            printf("%d,%d,%d,%d,%d,%d,%d,%llu,%llu,%llu,%llu\n", grids[g], c.M, c.N, c.nmma, c.nacc, c.a_tmem, c.chunk_wait, h[0], h[1], h[2], h[3]);
        }
    }
    int herr = 0;
    cudaMemcpy(&herr, d_err, sizeof(int), cudaMemcpyDeviceToHost);
    printf("err=%d\n", herr);
    return herr;
}
