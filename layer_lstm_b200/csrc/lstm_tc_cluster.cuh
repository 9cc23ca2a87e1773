// Cluster-level building blocks shared by the tensor-core recurrences
// (forward and BPTT): cluster rank and barrier, distributed-shared-memory
// addresses and asynchronous stores that complete on a remote mbarrier,
// bounded waits on a cluster-scope mbarrier and on a global group counter.
// Every wait gives up on the block's abort flag, on an error recorded
// anywhere in the grid, or after its time limit, recording LSTM_ERR_TIMEOUT.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "lstm_device.cuh"
#include "lstm_tc.cuh"

namespace lstm {

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Shared-memory address of the same offset in block `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Asynchronous 16-byte store into another block of the cluster; its bytes
// count against the transaction count of that block's mbarrier remote_bar,
// so the storing thread does not wait for it to land.
__device__ __forceinline__ void st_async_v4(uint32_t addr, float a, float b, float c, float d, uint32_t remote_bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d), "r"(remote_bar)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(tc::smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the partner's partial sums: gives up on this block's abort
// flag, on an error anywhere in the grid, or after timeout_ns.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, volatile int* abort, int* status,
                                                  uint64_t timeout_ns) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    uint32_t it = 0;
    while (!mbar_try_wait_cluster(bar, parity)) {
        if ((++it & 255u) == 0) {
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

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    while (!tc::mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > 100000000ull) break;
    }
}

__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
                 : "memory");
}

// 3-D TMA map of a bf16 [rows][cols] matrix seen as (k within a 64-wide
// chunk, row, chunk): a box {64, box_rows, box_chunks} lands the chunks one
// after another, each a 128-byte-swizzled [box_rows][64] tile.
bool make_map_bf16_chunks(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows,
                          int box_chunks);

// The same for a float32 [rows][cols] matrix and 32-wide chunks: a box
// {32, box_rows, box_chunks} lands 128-byte-swizzled [box_rows][32] tiles.
bool make_map_f32_chunks(CUtensorMap* map, const void* base, long long rows, long long cols, int box_rows,
                         int box_chunks);

}  // namespace lstm
