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

template <typename T>
__global__ void pack_ih_kernel(PackIhArgs a) {
    const int G = 4 * a.H;
    const long long total = (long long)a.D * G * a.in;
    T* wp = static_cast<T*>(a.wp);
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int k = (int)(e % a.in);
        const long long row = e / a.in;
        const int d = (int)(row / G), p = (int)(row % G);
        const int src = (p & 3) * a.H + (p >> 2);
        wp[e] = static_cast<const T*>(a.w[d])[(long long)src * a.in + k];
        if (k == 0) {
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

__global__ void pack_hh_bwd_kernel(PackHhBwdArgs a) {
    const int G = 4 * a.H;
    const long long total = (long long)a.D * a.nu * G * a.U;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int jl = (int)(e % a.U);
        long long r2 = e / a.U;
        const int r = (int)(r2 % G);
        r2 /= G;
        const int j = (int)(r2 % a.nu);
        const int d = (int)(r2 / a.nu);
        const int col = j * a.U + jl;
        a.out[e] = col < a.H ? a.w[d][(long long)r * a.H + col] : 0.f;
    }
}

inline int grid_for(long long total) {
    long long g = (total + 255) / 256;
    return (int)std::min<long long>(std::max<long long>(g, 1), 148LL * 16);
}

}  // namespace

cudaError_t launch_pack_ih(const PackIhArgs& a, cudaStream_t s) {
    const long long total = (long long)a.D * 4 * a.H * a.in;
    if (a.dt == DType::F32)
        pack_ih_kernel<float><<<grid_for(total), 256, 0, s>>>(a);
    else
        pack_ih_kernel<bf16><<<grid_for(total), 256, 0, s>>>(a);
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

cudaError_t launch_pack_hh_bwd(const PackHhBwdArgs& a, cudaStream_t s) {
    const long long total = (long long)a.D * a.nu * 4 * a.H * a.U;
    pack_hh_bwd_kernel<<<grid_for(total), 256, 0, s>>>(a);
    return cudaGetLastError();
}

// ==========================================================  block matvec
namespace {

// red[ks][r][b] = sum over k in slice ks of Wk[k*R + r] * Hs[b*Kp + k].
// R, Bs and Kp are multiples of 4.  Each thread owns 4 rows x 4 batch
// columns of one K slice and walks k four at a time (4 + 4 vector loads per
// 64 FMA); threads of a warp share batch columns so the h loads broadcast.
template <typename WT, typename HT>
__device__ __forceinline__ void block_matvec(const WT* __restrict__ Wk, int R,
                                             const HT* __restrict__ Hs, int Bs, int Kp, int KS,
                                             float* __restrict__ red) {
    const int nRT = R >> 2, nBT = Bs >> 2, nT = nRT * nBT;
    const int KL = (((Kp >> 2) + KS - 1) / KS) << 2;
    for (int it = threadIdx.x; it < nT * KS; it += blockDim.x) {
        const int tile = it % nT, ks = it / nT;
        const int rt = tile % nRT, bt = tile / nRT;
        const int k0 = ks * KL, k1 = min(Kp, k0 + KL);
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
        const WT* wp = Wk + rt * 4;
        const HT* hp = Hs + (size_t)bt * 4 * Kp;
#pragma unroll 2
        for (int k = k0; k < k1; k += 4) {
            float w[4][4], h[4][4];
#pragma unroll
            for (int q = 0; q < 4; ++q) load4(wp + (size_t)(k + q) * R, w[q]);
#pragma unroll
            for (int j = 0; j < 4; ++j) load4(hp + (size_t)j * Kp + k, h[j]);
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(w[q][i], h[j][q], acc[i][j]);
        }
        float* rp = red + ((size_t)ks * R + rt * 4) * Bs + bt * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            *reinterpret_cast<float4*>(rp + (size_t)i * Bs) =
                make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    }
}

// Four elements of T as one vector load/store.
template <typename T> struct Vec4;
template <> struct Vec4<float> {
    typedef float4 type;
    static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <> struct Vec4<bf16> {
    typedef uint2 type;
    static __device__ __forceinline__ uint2 zero() { return make_uint2(0u, 0u); }
};

// dst[bl*Kp + k] = src[bl*ld + k] for bl < nb, k < K; zeros for bl in
// [nb, Bs) and k in [K, Kp).  L1 is bypassed (the rows were written by other
// blocks during this kernel).  Loads are issued in groups of 8 per thread
// before their stores so that many L2 requests are in flight.
template <typename T>
__device__ __forceinline__ void copy_rows_to_smem(T* __restrict__ dst, int Kp, int Bs,
                                                  const T* __restrict__ src, size_t ld, int nb,
                                                  int K) {
    constexpr int UN = 8;
    const int tid = threadIdx.x, nth = blockDim.x;
    const bool vec = src != nullptr && (K & 3) == 0 && (ld & 3) == 0 &&
                     ((reinterpret_cast<uintptr_t>(src) & (4 * sizeof(T) - 1)) == 0);
    if (vec) {
        typedef typename Vec4<T>::type V;
        const int kv = Kp >> 2;
        const int total = Bs * kv;
        for (int base = tid; base < total; base += nth * UN) {
            V v[UN];
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                v[u] = Vec4<T>::zero();
                if (i < total) {
                    const int bl = i / kv, k4 = i % kv;
                    if (bl < nb) v[u] = __ldcg(reinterpret_cast<const V*>(src + bl * ld) + k4);
                }
            }
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                if (i < total) {
                    const int bl = i / kv, k4 = i % kv;
                    reinterpret_cast<V*>(dst + (size_t)bl * Kp)[k4] = v[u];
                }
            }
        }
    } else {
        const int total = Bs * Kp;
        for (int base = tid; base < total; base += nth * UN) {
            T v[UN];
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                v[u] = from_f<T>(0.f);
                if (i < total && src) {
                    const int bl = i / Kp, k = i % Kp;
                    if (bl < nb && k < K) v[u] = ld_cg(src + bl * ld + k);
                }
            }
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                if (i < total) dst[i] = v[u];
            }
        }
    }
}

__device__ __forceinline__ size_t align16(size_t x) { return (x + 15) & ~size_t(15); }
inline size_t align16h(size_t x) { return (x + 15) & ~size_t(15); }

inline int pick_ks(int R, int Bs, int Kp) {
    const int nT = (R / 4) * (Bs / 4);
    int ks = 1;
    while (nT * ks * 2 <= 256 && Kp / (ks * 2) >= 8) ks *= 2;
    return ks;
}

}  // namespace

// =========================================================  forward recurrence
//
// Grid: D x nbg x nu persistent blocks, launched cooperatively so that all are
// co-resident.  Block (d, bg, j) owns hidden units [j*U, j*U+U) of direction d
// (the 4U gate rows i,f,g,o of those units, resident in shared memory) for the
// batch rows of group bg.  Step s handles time t = s (forward direction) or
// T-1-s (reverse).  Per step a block gathers h_{t-1} of its batch rows from the
// layer's output sequence (written by the other blocks of its group in the
// previous step), forms W_hh h_{t-1} + Gx[t] (Gx holds W_ih x_t + b_ih + b_hh
// from the time-batched projection), applies the gates and the c/h update,
// writes h_t and arrives on the group counter.
namespace {

template <typename WT>
__global__ void __launch_bounds__(256, 1) fwd_rec_kernel(FwdRecArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const RecPlan& p = a.p;
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int Hp = (H + 3) & ~3;
    const int U = p.U, R = 4 * U, Bs = p.Bs, KS = p.KS;
    WT* Ws = reinterpret_cast<WT*>(smem);                              // [Hp][R]
    size_t off = align16((size_t)Hp * R * sizeof(WT));
    WT* hs = reinterpret_cast<WT*>(smem + off);                        // [Bs][Hp]
    off += align16((size_t)Hp * Bs * sizeof(WT));
    float* red = reinterpret_cast<float*>(smem + off);                 // [KS][R][Bs]
    off += align16((size_t)KS * R * Bs * sizeof(float));
    float* cs = reinterpret_cast<float*>(smem + off);                  // [U][Bg]

    const int j = blockIdx.x % p.nu;
    const int bg = (blockIdx.x / p.nu) % p.nbg;
    const int d = blockIdx.x / (p.nu * p.nbg);
    const int u0 = j * U, nU = min(U, H - u0);
    const int b0 = bg * p.Bg, nB = min(p.Bg, B - b0);
    const WT* wsrc = static_cast<const WT*>(a.wpk) + ((size_t)d * p.nu + j) * Hp * R;
    const WT* h0 = static_cast<const WT*>(a.h0);
    WT* hseq = static_cast<WT*>(a.hseq);
    WT* out = static_cast<WT*>(a.out);
    WT* h_n = static_cast<WT*>(a.h_n);
    const int tid = threadIdx.x, nth = blockDim.x;

    {   // resident weights: a plain contiguous copy of this block's slice
        typedef typename Vec4<WT>::type V;
        const int nv = Hp * R / 4;
        const V* s4 = reinterpret_cast<const V*>(wsrc);
        V* d4 = reinterpret_cast<V*>(Ws);
        for (int i = tid; i < nv; i += nth) d4[i] = s4[i];
    }
    for (int i = tid; i < U * p.Bg; i += nth) {
        const int ul = i / p.Bg, bl = i % p.Bg;
        float c = 0.f;
        if (a.c0 && ul < nU && bl < nB) c = a.c0[((size_t)d * B + b0 + bl) * H + u0 + ul];
        cs[i] = c;
    }
    __syncthreads();
    if (nB <= 0) return;   // plans never leave a group empty

    unsigned* ctr = a.ctr + d * p.nbg + bg;
    const size_t ldseq = (size_t)D * H;
    const int nb0 = min(Bs, nB);
    const int np0 = nU * nb0;          // pairs of the first batch sub-tile
    for (int s = 0; s < T; ++s) {
        const int t = d == 0 ? s : T - 1 - s;
        const int tp = d == 0 ? t - 1 : t + 1;
        // Gx of this thread's (unit, row) pairs in the first sub-tile does not
        // depend on other blocks: fetch it before waiting.
        float4 gxp[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int i = tid + q * nth;
            gxp[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (i < np0) {
                const int ul = i % nU, bl = i / nU;
                gxp[q] = *reinterpret_cast<const float4*>(
                    a.gx + ((size_t)t * B + b0 + bl) * (size_t)(D * G) + (size_t)d * G + 4 * (u0 + ul));
            }
        }
        if (s > 0 && p.nu > 1) {
            if (!block_wait_geq(ctr, (unsigned)(p.nu * s), a.status, a.timeout_ns)) return;
        }
        for (int bs0 = 0; bs0 < nB; bs0 += Bs) {
            const int nb = min(Bs, nB - bs0);
            const WT* src;
            size_t ld;
            if (s == 0) {
                src = h0 ? h0 + ((size_t)d * B + b0 + bs0) * H : nullptr;
                ld = H;
            } else {
                src = hseq + ((size_t)tp * B + b0 + bs0) * ldseq + (size_t)d * H;
                ld = ldseq;
            }
            copy_rows_to_smem(hs, Hp, Bs, src, ld, nb, H);
            __syncthreads();
            block_matvec(Ws, R, hs, Bs, Hp, KS, red);
            __syncthreads();
            for (int i = tid, q = 0; i < nU * nb; i += nth, ++q) {
                const int ul = i % nU, bl = i / nU;
                const int b = b0 + bs0 + bl, u = u0 + ul;
                float4 gxv;
                if (bs0 == 0 && q < 2) {
                    gxv = gxp[q];
                } else {
                    gxv = *reinterpret_cast<const float4*>(
                        a.gx + ((size_t)t * B + b) * (size_t)(D * G) + (size_t)d * G + 4 * u);
                }
                float pre[4] = {gxv.x, gxv.y, gxv.z, gxv.w};
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    float acc = 0.f;
                    for (int ks = 0; ks < KS; ++ks) acc += red[((size_t)ks * R + 4 * ul + g) * Bs + bl];
                    pre[g] += acc;
                }
                const float ig = sigmoidf_(pre[0]);
                const float fg = sigmoidf_(pre[1]);
                const float gg = tanhf(pre[2]);
                const float og = sigmoidf_(pre[3]);
                float& cref = cs[ul * p.Bg + bs0 + bl];
                const float c = fg * cref + ig * gg;
                cref = c;
                const float h = og * tanhf(c);
                const WT hv = from_f<WT>(h);
                hseq[((size_t)t * B + b) * ldseq + (size_t)d * H + u] = hv;
                if (out) out[(size_t)t * a.out_st + (size_t)b * a.out_sb + (size_t)d * H + u] = hv;
                if (a.act) {
                    *reinterpret_cast<float4*>(a.act + (((size_t)d * T + t) * B + b) * G + 4 * u) =
                        make_float4(ig, fg, gg, og);
                    a.cst[(((size_t)d * T + t) * B + b) * H + u] = c;
                }
                if (s == T - 1) {
                    h_n[((size_t)d * B + b) * H + u] = hv;
                    a.c_n[((size_t)d * B + b) * H + u] = c;
                }
            }
            __syncthreads();
        }
        if (p.nu > 1 && s + 1 < T) block_arrive(ctr);
    }
}

}  // namespace

RecPlan plan_fwd_rec(int H, int B, int D, DType dt, int num_sms, size_t smem_max) {
    const size_t es = dtype_size(dt);
    const int Hp = (H + 3) & ~3;
    RecPlan best{};
    double best_cost = 1e300;
    const int Us[] = {1, 2, 4, 8, 16, 32, 64};
    for (int U : Us) {
        const int nu = (H + U - 1) / U;
        if (U > 1 && (U / 2) >= H) break;
        for (int nbg = 1; nbg <= std::max(B, 1); ++nbg) {
            const int ctas = D * nbg * nu;
            if (ctas > num_sms) break;
            const int Bg = (B + nbg - 1) / nbg;
            if (nbg > 1 && (nbg - 1) * Bg >= B) continue;   // a group would be empty
            int Bs = std::min(((Bg + 3) / 4) * 4, 64);
            if (Bs < 4) Bs = 4;
            RecPlan pl{};
            bool ok = false;
            for (; Bs >= 4; Bs -= 4) {
                const int R = 4 * U;
                const int KS = pick_ks(R, Bs, Hp);
                const size_t smem = align16h((size_t)Hp * R * es) + align16h((size_t)Hp * Bs * es) +
                                    align16h((size_t)KS * R * Bs * 4) + align16h((size_t)U * Bg * 4);
                if (smem <= smem_max) {
                    pl = RecPlan{nbg, Bg, nu, U, Bs, KS, 256, smem, ctas};
                    ok = true;
                    break;
                }
            }
            if (!ok) continue;
            const int nsub = (Bg + pl.Bs - 1) / pl.Bs;
            // per-step time estimate in SM cycles: FFMA work + per-sub-tile
            // latency (copy, two barriers, epilogue) + group synchronisation
            const double fma = 4.0 * U * nsub * pl.Bs * (double)Hp;
            const double cost = fma / 96.0 + nsub * 1500.0 + (nu > 1 ? 2500.0 : 0.0) +
                                (double)ctas * 1e-3;
            if (cost < best_cost) {
                best_cost = cost;
                best = pl;
            }
        }
    }
    return best;
}

cudaError_t launch_fwd_rec(const FwdRecArgs& a, cudaStream_t s) {
    FwdRecArgs args = a;
    void* params[] = {&args};
    const void* fn = a.dt == DType::F32 ? reinterpret_cast<const void*>(&fwd_rec_kernel<float>)
                                        : reinterpret_cast<const void*>(&fwd_rec_kernel<bf16>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)a.p.smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchCooperativeKernel(fn, dim3(a.p.ctas), dim3(a.p.threads), params, a.p.smem, s);
}

// =========================================================  BPTT recurrence
//
// Grid: D x nbg x nu persistent blocks.  Block (d, bg, j) owns the gradient
// w.r.t. h of hidden units J = [j*U, j*U+U) for the batch rows of group bg and
// keeps the columns J of W_hh (all 4H rows) resident.  Step s (s = 0..T-1)
// handles time t = T-1-s (forward direction) or s (reverse):
//   dh_t  = dy_t + dh_rec,   dh_rec = sum_r W_hh[r][J] * da_{t+1}[r]
//   (gate derivatives, dc carry) -> da_t, written to dG (all 4H rows of a
//   block's units) and read by every block of the group at step s+1.
// Step T only forms dh_rec from da at the last time, which is dh0.
namespace {

struct BwdPre {
    float dy, c, cp;
    float4 act;
};

__device__ __forceinline__ BwdPre bwd_fetch(const BwdRecArgs& a, int d, int t, int b, int jj) {
    const int H = a.H, B = a.B, T = a.T, G = 4 * H;
    BwdPre r;
    r.dy = a.dy[(size_t)t * a.dy_st + (size_t)b * a.dy_sb + (size_t)d * H + jj];
    r.act = *reinterpret_cast<const float4*>(a.act + (((size_t)d * T + t) * B + b) * G + 4 * jj);
    r.c = a.cst[(((size_t)d * T + t) * B + b) * H + jj];
    const int tpf = d == 0 ? t - 1 : t + 1;
    const bool has_prev = d == 0 ? (t >= 1) : (t + 1 < T);
    r.cp = has_prev ? a.cst[(((size_t)d * T + tpf) * B + b) * H + jj]
                    : (a.c0 ? a.c0[((size_t)d * B + b) * H + jj] : 0.f);
    return r;
}

__global__ void __launch_bounds__(256, 1) bwd_rec_kernel(BwdRecArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const RecPlan& p = a.p;
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int U = p.U, Bs = p.Bs, KS = p.KS;
    float* Wt = reinterpret_cast<float*>(smem);                      // [G][U]
    size_t off = align16((size_t)G * U * 4);
    float* das = reinterpret_cast<float*>(smem + off);               // [Bs][G]
    off += align16((size_t)G * Bs * 4);
    float* red = reinterpret_cast<float*>(smem + off);               // [KS][U][Bs]
    off += align16((size_t)KS * U * Bs * 4);
    float* dcs = reinterpret_cast<float*>(smem + off);               // [U][Bg]
    off += align16((size_t)U * p.Bg * 4);
    float* dbacc = reinterpret_cast<float*>(smem + off);             // [4][U][Bg]

    const int j = blockIdx.x % p.nu;
    const int bg = (blockIdx.x / p.nu) % p.nbg;
    const int d = blockIdx.x / (p.nu * p.nbg);
    const int j0 = j * U, nU = min(U, H - j0);
    const int b0 = bg * p.Bg, nB = min(p.Bg, B - b0);
    const int tid = threadIdx.x, nth = blockDim.x;
    {
        const float4* s4 = reinterpret_cast<const float4*>(a.wt + ((size_t)d * p.nu + j) * G * U);
        float4* d4 = reinterpret_cast<float4*>(Wt);
        for (int i = tid; i < G * U / 4; i += nth) d4[i] = s4[i];
    }
    for (int i = tid; i < U * p.Bg; i += nth) {
        const int ul = i / p.Bg, bl = i % p.Bg;
        float dc = 0.f;
        if (a.grad_cn && ul < nU && bl < nB) dc = a.grad_cn[((size_t)d * B + b0 + bl) * H + j0 + ul];
        dcs[i] = dc;
    }
    for (int i = tid; i < 4 * U * p.Bg; i += nth) dbacc[i] = 0.f;
    __syncthreads();
    if (nB <= 0) return;

    unsigned* ctr = a.ctr + d * p.nbg + bg;
    const size_t ldg = (size_t)D * G;
    const int nb0 = min(Bs, nB);
    const int np0 = nU * nb0;
    for (int s = 0; s <= T; ++s) {
        const int t = d == 0 ? T - 1 - s : s;            // time handled at this step (s < T)
        const int tl = d == 0 ? t + 1 : t - 1;           // time handled at step s-1
        BwdPre pre[2];
        if (s < T) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int i = tid + q * nth;
                if (i < np0) pre[q] = bwd_fetch(a, d, t, b0 + i / nU, j0 + i % nU);
            }
        }
        if (s > 0 && p.nu > 1) {
            if (!block_wait_geq(ctr, (unsigned)(p.nu * s), a.status, a.timeout_ns)) return;
        }
        for (int bs0 = 0; bs0 < nB; bs0 += Bs) {
            const int nb = min(Bs, nB - bs0);
            if (s > 0) {
                copy_rows_to_smem(das, G, Bs, a.dG + ((size_t)tl * B + b0 + bs0) * ldg + (size_t)d * G,
                                  ldg, nb, G);
                __syncthreads();
                block_matvec(Wt, U, das, Bs, G, KS, red);
                __syncthreads();
            }
            for (int i = tid, q = 0; i < nU * nb; i += nth, ++q) {
                const int ul = i % nU, bl = i / nU;
                const int b = b0 + bs0 + bl, jj = j0 + ul;
                const size_t sidx = ((size_t)d * B + b) * H + jj;
                float dhrec = 0.f;
                if (s > 0) {
                    for (int ks = 0; ks < KS; ++ks) dhrec += red[((size_t)ks * U + ul) * Bs + bl];
                } else if (a.grad_hn) {
                    dhrec = a.grad_hn[sidx];
                }
                float& dcref = dcs[ul * p.Bg + bs0 + bl];
                if (s == T) {
                    a.dh0[sidx] = dhrec;
                    a.dc0[sidx] = dcref;
                    continue;
                }
                const BwdPre v = (bs0 == 0 && q < 2) ? pre[q] : bwd_fetch(a, d, t, b, jj);
                const float ig = v.act.x, fg = v.act.y, gg = v.act.z, og = v.act.w;
                const float dh = v.dy + dhrec;
                const float th = tanhf(v.c);
                const float dc = dcref + dh * og * (1.f - th * th);
                const float da_i = dc * gg * ig * (1.f - ig);
                const float da_f = dc * v.cp * fg * (1.f - fg);
                const float da_g = dc * ig * (1.f - gg * gg);
                const float da_o = dh * th * og * (1.f - og);
                dcref = dc * fg;
                float* dgp = a.dG + ((size_t)t * B + b) * ldg + (size_t)d * G + jj;
                dgp[0] = da_i;
                dgp[H] = da_f;
                dgp[2 * H] = da_g;
                dgp[3 * H] = da_o;
                float* dba = dbacc + (size_t)ul * p.Bg + bs0 + bl;
                dba[0] += da_i;
                dba[(size_t)U * p.Bg] += da_f;
                dba[(size_t)2 * U * p.Bg] += da_g;
                dba[(size_t)3 * U * p.Bg] += da_o;
            }
            __syncthreads();
        }
        if (p.nu > 1 && s < T) block_arrive(ctr);
    }
    // bias-gradient partial of this block: sum over its batch rows, fixed order
    for (int i = tid; i < 4 * nU; i += nth) {
        const int q = i / nU, ul = i % nU;
        const float* row = dbacc + ((size_t)q * U + ul) * p.Bg;
        float sum = 0.f;
        for (int bl = 0; bl < nB; ++bl) sum += row[bl];
        a.dbpart[((size_t)d * p.nbg + bg) * G + (size_t)q * H + j0 + ul] = sum;
    }
}

__global__ void db_reduce_kernel(DbArgs a) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= a.D * a.G) return;
    const int d = e / a.G, r = e % a.G;
    float sum = 0.f;
    for (int g = 0; g < a.nbg; ++g) sum += a.dbpart[((size_t)d * a.nbg + g) * a.G + r];
    a.db_ih[d][r] = sum;
    a.db_hh[d][r] = sum;
}

template <typename T>
__global__ void seq_copy_kernel(SeqCopyArgs a) {
    const long long total = (long long)a.T * a.B * a.W;
    const T* src = static_cast<const T*>(a.src);
    T* dst = static_cast<T*>(a.dst);
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int w = (int)(e % a.W);
        const long long tb = e / a.W;
        const int b = (int)(tb % a.B), t = (int)(tb / a.B);
        dst[t * a.d_st + b * a.d_sb + w] = src[t * a.s_st + b * a.s_sb + w];
    }
}

}  // namespace

RecPlan plan_bwd_rec(int H, int B, int D, int num_sms, size_t smem_max) {
    const int G = 4 * H;
    RecPlan best{};
    double best_cost = 1e300;
    const int Us[] = {4, 8, 16, 32};
    for (int U : Us) {
        const int nu = (H + U - 1) / U;
        if (U > 4 && (U / 2) >= H) break;
        for (int nbg = 1; nbg <= std::max(B, 1); ++nbg) {
            const int ctas = D * nbg * nu;
            if (ctas > num_sms) break;
            const int Bg = (B + nbg - 1) / nbg;
            if (nbg > 1 && (nbg - 1) * Bg >= B) continue;
            int Bs = std::min(((Bg + 3) / 4) * 4, 32);
            if (Bs < 4) Bs = 4;
            RecPlan pl{};
            bool ok = false;
            for (; Bs >= 4; Bs -= 4) {
                const int KS = pick_ks(U, Bs, G);
                const size_t smem = align16h((size_t)G * U * 4) + align16h((size_t)G * Bs * 4) +
                                    align16h((size_t)KS * U * Bs * 4) + align16h((size_t)U * Bg * 4) +
                                    align16h((size_t)4 * U * Bg * 4);
                if (smem <= smem_max) {
                    pl = RecPlan{nbg, Bg, nu, U, Bs, KS, 256, smem, ctas};
                    ok = true;
                    break;
                }
            }
            if (!ok) continue;
            const int nsub = (Bg + pl.Bs - 1) / pl.Bs;
            const double fma = (double)U * nsub * pl.Bs * (double)G;
            const double cost = fma / 96.0 + nsub * 1500.0 + (nu > 1 ? 2500.0 : 0.0) +
                                (double)ctas * 1e-3;
            if (cost < best_cost) {
                best_cost = cost;
                best = pl;
            }
        }
    }
    return best;
}

cudaError_t launch_bwd_rec(const BwdRecArgs& a, cudaStream_t s) {
    BwdRecArgs args = a;
    void* params[] = {&args};
    const void* fn = reinterpret_cast<const void*>(&bwd_rec_kernel);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)a.p.smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchCooperativeKernel(fn, dim3(a.p.ctas), dim3(a.p.threads), params, a.p.smem, s);
}

cudaError_t launch_db_reduce(const DbArgs& a, cudaStream_t s) {
    const int n = a.D * a.G;
    db_reduce_kernel<<<(n + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_seq_copy(const SeqCopyArgs& a, cudaStream_t s) {
    const long long total = (long long)a.T * a.B * a.W;
    if (total <= 0) return cudaSuccess;
    if (a.dt == DType::F32)
        seq_copy_kernel<float><<<grid_for(total), 256, 0, s>>>(a);
    else
        seq_copy_kernel<bf16><<<grid_for(total), 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lstm
