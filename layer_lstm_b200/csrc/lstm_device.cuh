// Device-side helpers shared by the LSTM kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lstm_internal.h"

namespace lstm {

// Kernel-side status codes written to the workspace status word; the values
// match lstm_status in include/lstm.h.
constexpr int kStatusOk = 0;
constexpr int kStatusTimeout = 5;

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// Four consecutive elements to float (16-byte aligned for float, 8 for bf16).
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
    const float4 q = *reinterpret_cast<const float4*>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(&q.x);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&q.y);
    const float2 fa = __bfloat1622float2(a), fb = __bfloat1622float2(b);
    v[0] = fa.x; v[1] = fa.y; v[2] = fb.x; v[3] = fb.y;
}

// Load that bypasses L1 (the value may have been written by another SM
// during this kernel).
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }
__device__ __forceinline__ bf16 ld_cg(const bf16* p) {
    unsigned short r;
    asm volatile("ld.global.cg.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return __ushort_as_bfloat16(r);
}

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ int ld_volatile(const int* p) {
    return *reinterpret_cast<const volatile int*>(p);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Per-step timeline (instrumentation): the calling thread stamps event e of
// step s when tracing is on (trace non-null) and `who` holds.
__device__ __forceinline__ void trace_mark(unsigned long long* trace, bool who, int s, int e) {
    if (trace != nullptr && who && s < kTraceSteps) trace[(size_t)s * kTraceEvents + e] = globaltimer_ns();
}

// Block-wide arrival on a counter: every thread's prior global writes are
// made visible at GPU scope before the count moves.
// *ctr += v with release semantics at GPU scope: everything the block wrote
// before the preceding barrier is visible to whoever acquires the new value.
__device__ __forceinline__ void red_release_add(unsigned* ctr, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(ctr), "r"(v) : "memory");
}

__device__ __forceinline__ void block_arrive(unsigned* ctr) {
    __syncthreads();
    if (threadIdx.x == 0) red_release_add(ctr, 1u);
}

// Block-wide bounded wait until *ctr >= target.  Returns false (for every
// thread of the block) when the wait gave up or another block already
// reported a failure; the first block to give up records kStatusTimeout.
__device__ __forceinline__ bool block_wait_geq(const unsigned* ctr, unsigned target, int* status,
                                               uint64_t timeout_ns) {
    __shared__ int ok_s;
    if (threadIdx.x == 0) {
        int ok = 1;
        if (ld_acquire(ctr) < target) {
            const uint64_t t0 = globaltimer_ns();
            unsigned it = 0;
            while (ld_acquire(ctr) < target) {
                if ((++it & 63u) == 0) {
                    if (ld_volatile(status) != kStatusOk) { ok = 0; break; }
                    if (globaltimer_ns() - t0 > timeout_ns) {
                        atomicCAS(status, kStatusOk, kStatusTimeout);
                        ok = 0;
                        break;
                    }
                }
            }
        }
        ok_s = ok;   // the acquire loads above order what follows
    }
    __syncthreads();
    return ok_s != 0;
}

__device__ __forceinline__ float sigmoidf_(float z) { return 1.0f / (1.0f + expf(-z)); }

}  // namespace lstm
