// CUDA-core (FFMA) kernels of the LSTM path: weight packing, a strided GEMM
// used for small or odd shapes, the persistent forward recurrence, the
// persistent BPTT gate-gradient recurrence, and small reductions/copies.
//
// The cell and its gradient follow the warp_nn "Long Short-Term Memory (LSTM)"
// page (equation block; i, f, g, o row stacking of the "Learnable parameters"
// table).  The backward is reverse-mode differentiation of the unrolled time
// loop ("LSTM Forward Computation", Loop Unroll) with weight gradients summed
// over all steps (pulsatrix LSTMModule, backward()).
#include <algorithm>

#include "lstm_device.cuh"
#include "lstm_internal.h"

namespace lstm {

// =====================================================================  GEMM
namespace {

template <typename TA, typename TB, typename TC>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmArgs g) {
    constexpr int BM = 64, BN = 64, BK = 16;
    __shared__ __align__(16) float As[BK][BM + 4];
    __shared__ __align__(16) float Bs[BK][BN + 4];
    const TA* A = static_cast<const TA*>(g.A);
    const TB* B = static_cast<const TB*>(g.B);
    const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const bool a_kc = g.sAk == 1;
    const bool b_nc = g.sBn == 1;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    for (int k0 = 0; k0 < g.K; k0 += BK) {
        for (int e = tid; e < BM * BK; e += 256) {
            const int mm = a_kc ? e / BK : e % BM;
            const int kk = a_kc ? e % BK : e / BM;
            const int m = m0 + mm, k = k0 + kk;
            float v = 0.f;
            if (m < g.M && k < g.K) v = to_f(A[(long long)m * g.sAm + (long long)k * g.sAk]);
            As[kk][mm] = v;
        }
        for (int e = tid; e < BK * BN; e += 256) {
            const int nn = b_nc ? e % BN : e / BK;
            const int kk = b_nc ? e / BN : e % BK;
            const int n = n0 + nn, k = k0 + kk;
            float v = 0.f;
            if (n < g.N && k < g.K) v = to_f(B[(long long)k * g.sBk + (long long)n * g.sBn]);
            Bs[kk][nn] = v;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float a[4], b[4];
            load4(&As[kk][ty * 4], a);
            load4(&Bs[kk][tx * 4], b);
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    TC* C = static_cast<TC*>(g.C);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= g.M) continue;
        long long row = m;
        if (g.remap_T > 0) {            // m = b*T + t  ->  t*B + b
            const int T = g.remap_T;
            row = (long long)(m % T) * g.remap_B + m / T;
        } else if (g.remap_T < 0) {     // m = t*B + b  ->  b*T + t
            const int T = -g.remap_T;
            row = (long long)(m % g.remap_B) * T + m / g.remap_B;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = n0 + tx * 4 + j;
            if (n >= g.N) continue;
            float v = acc[i][j] + (g.bias ? g.bias[n] : 0.f);
            TC* cp = C + row * g.ldc + n;
            if (g.accumulate) v += to_f(*cp);
            *cp = from_f<TC>(v);
        }
    }
}

template <typename TA, typename TB>
cudaError_t gemm_dispatch_c(const GemmArgs& g, cudaStream_t s) {
    dim3 grid((g.N + 63) / 64, (g.M + 63) / 64);
    if (g.tc == DType::F32)
        gemm_simt_kernel<TA, TB, float><<<grid, 256, 0, s>>>(g);
    else
        gemm_simt_kernel<TA, TB, bf16><<<grid, 256, 0, s>>>(g);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s) {
    if (g.M <= 0 || g.N <= 0) return cudaSuccess;
    if (g.ta == DType::F32 && g.tb == DType::F32) return gemm_dispatch_c<float, float>(g, s);
    if (g.ta == DType::BF16 && g.tb == DType::BF16) return gemm_dispatch_c<bf16, bf16>(g, s);
    if (g.ta == DType::F32 && g.tb == DType::BF16) return gemm_dispatch_c<float, bf16>(g, s);
    return gemm_dispatch_c<bf16, float>(g, s);
}

// ==================================================================  packing
namespace {

// One block per packed row (grid-stride over rows), its threads over the
// row's contiguous columns: no per-element division.
template <typename T>
__global__ void pack_ih_kernel(PackIhArgs a) {
    const int G = 4 * a.H;
    for (int row = blockIdx.x; row < a.D * G; row += gridDim.x) {
        const int d = row / G, p = row - d * G;
        const int src = (p & 3) * a.H + (p >> 2);
        const T* w = static_cast<const T*>(a.w[d]) + (size_t)src * a.in;
        T* wp = static_cast<T*>(a.wp) + (size_t)row * a.in;
        for (int k = threadIdx.x; k < a.in; k += blockDim.x) wp[k] = w[k];
        if (threadIdx.x == 0) {
            float b = 0.f;
            if (a.b_ih[d]) b += to_f(static_cast<const T*>(a.b_ih[d])[src]);
            if (a.b_hh[d]) b += to_f(static_cast<const T*>(a.b_hh[d])[src]);
            a.bias_p[row] = b;
        }
    }
}

template <typename T>
__global__ void pack_hh_fwd_kernel(PackHhFwdArgs a) {
    const int R = 4 * a.U;
    const int Hp = (a.H + 3) & ~3;
    const long long total = (long long)a.D * a.nu * Hp * R;
    T* out = static_cast<T*>(a.out);
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int rl = (int)(e % R);
        long long r2 = e / R;
        const int k = (int)(r2 % Hp);
        r2 /= Hp;
        const int j = (int)(r2 % a.nu);
        const int d = (int)(r2 / a.nu);
        const int u = j * a.U + (rl >> 2);
        T v = from_f<T>(0.f);
        if (u < a.H && k < a.H) v = static_cast<const T*>(a.w[d])[((long long)(rl & 3) * a.H + u) * a.H + k];
        out[e] = v;
    }
}

inline int grid_for(long long total) {
    long long g = (total + 255) / 256;
    return (int)std::min<long long>(std::max<long long>(g, 1), 148LL * 16);
}

}  // namespace

cudaError_t launch_pack_ih(const PackIhArgs& a, cudaStream_t s) {
    const int rows = a.D * 4 * a.H;
    if (rows <= 0) return cudaSuccess;
    const int grid = std::min(rows, 148 * 16);
    if (a.dt == DType::F32)
        pack_ih_kernel<float><<<grid, 256, 0, s>>>(a);
    else
        pack_ih_kernel<bf16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_pack_hh_fwd(const PackHhFwdArgs& a, cudaStream_t s) {
    const long long total = (long long)a.D * a.nu * ((a.H + 3) & ~3) * 4 * a.U;
    if (a.dt == DType::F32)
        pack_hh_fwd_kernel<float><<<grid_for(total), 256, 0, s>>>(a);
    else
        pack_hh_fwd_kernel<bf16><<<grid_for(total), 256, 0, s>>>(a);
    return cudaGetLastError();
}

namespace {

__global__ void db_reduce_kernel(DbArgs a) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= a.D * a.G) return;
    const int d = e / a.G, r = e % a.G;
    float sum = 0.f;
    for (int g = 0; g < a.nbg; ++g) sum += a.dbpart[((size_t)d * a.nbg + g) * a.G + r];
    a.db_ih[d][r] = sum;
    a.db_hh[d][r] = sum;
}

// One block per (t, b) row (grid-stride over rows), its threads over the
// row's W contiguous elements: no per-element division.
template <typename T>
__global__ void seq_copy_kernel(SeqCopyArgs a) {
    const T* src = static_cast<const T*>(a.src);
    T* dst = static_cast<T*>(a.dst);
    for (int tb = blockIdx.x; tb < a.T * a.B; tb += gridDim.x) {
        const int t = tb / a.B, b = tb - t * a.B;
        const T* s = src + t * a.s_st + b * a.s_sb;
        T* o = dst + t * a.d_st + b * a.d_sb;
        for (int w = threadIdx.x; w < a.W; w += blockDim.x) o[w] = s[w];
    }
}

// Philox4x64-10, Salmon, Moraes, Dror, Shaw (2011), "Parallel random numbers:
// as easy as 1, 2, 3": ten rounds of
//   (R0, R1, R2, R3) -> (hi(M1 R2) ^ R1 ^ K0, lo(M1 R2), hi(M0 R0) ^ R3 ^ K1, lo(M0 R0))
// with the key advanced by the Weyl constants after each round.
__device__ __forceinline__ void philox4x64_10(uint64_t c[4], uint64_t k0, uint64_t k1) {
    const uint64_t M0 = 0xD2E7470EE14C6C93ull, M1 = 0xCA5A826395121157ull;
    const uint64_t W0 = 0x9E3779B97F4A7C15ull, W1 = 0xBB67AE8584CAA73Bull;
#pragma unroll
    for (int r = 0; r < 10; ++r) {
        const uint64_t hi0 = __umul64hi(M0, c[0]), lo0 = M0 * c[0];
        const uint64_t hi1 = __umul64hi(M1, c[2]), lo1 = M1 * c[2];
        const uint64_t n0 = hi1 ^ c[1] ^ k0, n2 = hi0 ^ c[3] ^ k1;
        c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
        k0 += W0;
        k1 += W1;
    }
}

// One Philox block per thread iteration: four consecutive elements.
template <typename T>
__global__ void dropout_kernel(DropoutArgs a) {
    const T* src = static_cast<const T*>(a.src);
    T* dst = static_cast<T*>(a.dst);
    const long long nblk = (a.n + 3) / 4;
    for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < nblk;
         q += (long long)gridDim.x * blockDim.x) {
        uint64_t w[4] = {(uint64_t)q, 0, 0, 0};
        philox4x64_10(w, a.seed, (uint64_t)a.layer);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const long long e = 4 * q + j;
            if (e >= a.n) break;
            const bool keep = (w[j] >> 11) >= a.thresh;
            dst[e] = from_f<T>(keep ? to_f(src[e]) * a.scale : 0.f);
        }
    }
}

// dst[i] = src[i] converted (float <-> bf16, round to nearest even)
template <typename S, typename D>
__global__ void convert_kernel(const S* __restrict__ src, D* __restrict__ dst, long long n) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x)
        dst[i] = from_f<D>(to_f(src[i]));
}

}  // namespace

cudaError_t launch_convert(const void* src, DType st, void* dst, DType dt, long long n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    if (st == DType::BF16 && dt == DType::F32)
        convert_kernel<<<grid_for(n), 256, 0, s>>>(static_cast<const bf16*>(src), static_cast<float*>(dst), n);
    else if (st == DType::F32 && dt == DType::BF16)
        convert_kernel<<<grid_for(n), 256, 0, s>>>(static_cast<const float*>(src), static_cast<bf16*>(dst), n);
    else
        return cudaMemcpyAsync(dst, src, (size_t)n * dtype_size(st), cudaMemcpyDeviceToDevice, s);
    return cudaGetLastError();
}

cudaError_t launch_dropout(const DropoutArgs& a, cudaStream_t s) {
    if (a.n <= 0) return cudaSuccess;
    const long long nblk = (a.n + 3) / 4;
    if (a.dt == DType::F32)
        dropout_kernel<float><<<grid_for(nblk), 256, 0, s>>>(a);
    else
        dropout_kernel<bf16><<<grid_for(nblk), 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_db_reduce(const DbArgs& a, cudaStream_t s) {
    const int n = a.D * a.G;
    db_reduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_seq_copy(const SeqCopyArgs& a, cudaStream_t s) {
    const long long rows = (long long)a.T * a.B;
    if (rows <= 0 || a.W <= 0) return cudaSuccess;
    const int grid = (int)std::min<long long>(rows, 148LL * 16);
    if (a.dt == DType::F32)
        seq_copy_kernel<float><<<grid, 256, 0, s>>>(a);
    else
        seq_copy_kernel<bf16><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lstm
