// Persistent recurrences on the CUDA cores (FFMA): the LSTM forward time loop
// and the BPTT gate-gradient time loop.
//
// Cell: warp_nn "Long Short-Term Memory (LSTM)" page, equation block
// (i, f, g, o; c' = f*c + i*g; h' = o*tanh(c')).  Backward: reverse-mode
// differentiation of the unrolled loop ("LSTM Forward Computation", Loop
// Unroll), weight gradients summed over all steps (pulsatrix LSTMModule,
// backward()).
//
// Both kernels run one cooperative grid of D x nbg x nu blocks: direction d,
// batch group bg (rows [bg*Bg, bg*Bg+Bg)), and unit slice j (hidden units
// [j*U, j*U+U)).  A block keeps the 4U rows of W_hh that belong to its units
// in shared memory for the whole sequence.  Blocks of one (d, bg) group meet
// once per step on a counter (bounded wait, see lstm_device.cuh).
//
//  forward  step: gather h_{t-1} of the group's rows from the exchange
//                 buffer hT[d][t][bg][k][bl] (group-major and k-major, so the
//                 group's tile is one contiguous block fetched with a single
//                 bulk async copy), a = W_slice h + Gx[t], gates, c/h update,
//                 write h_t (exchange, layer output, user output).
//  backward step: dh = dy_t + dh_rec for the block's units, gate derivatives
//                 and the dc carry -> da_t (the block's 4U gate rows); the
//                 block multiplies its own rows into a partial
//                 dh_{t-1}[b][0..H) = sum_{r in block} W_hh[r][:] da_t[r]
//                 and the owners of each unit add the nu partials in a fixed
//                 order after the step's barrier (a reduce-scatter whose
//                 traffic equals the forward's all-gather of h).
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "lstm_device.cuh"
#include "lstm_internal.h"
#include "lstm_tc.cuh"

namespace lstm {
namespace {

__device__ __forceinline__ size_t align16(size_t x) { return (x + 15) & ~size_t(15); }
inline size_t align16h(size_t x) { return (x + 15) & ~size_t(15); }

// C[r][n] = sum_k A[k*lda + r] * X[k*ldx + n] for r < R, n < N, k < K, with
// R and K multiples of 4 and N a multiple of TN (4 or 8).  Each thread
// computes a 4 x TN register tile over one of KS K-slices and hands it to
// st(ks, r0, n0, acc).  Lanes of a warp cover a wr x wn block of tiles of
// the same K-slice (wn tile columns, at most 128 contiguous bytes of X per
// load; wr = 32 / wn tile rows, contiguous in A), so shared-memory loads of
// a warp touch few wavefronts and no lane is idle while tiles remain.
template <int TN>
__host__ __device__ constexpr int tile_cols_wn(int nNT) {
    return nNT >= 128 / (4 * TN) ? 128 / (4 * TN) : (nNT >= 4 ? 4 : (nNT >= 2 ? 2 : 1));
}

// c0 += a * b0, c1 += a * b1 as one packed instruction (two IEEE fused
// multiply-adds, each rounded exactly as fmaf).
__device__ __forceinline__ void ffma2(float& c0, float& c1, float a, float b0, float b1) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %2};\n\tmov.b64 rb, {%3, %4};\n\tmov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(c0), "+f"(c1)
        : "f"(a), "f"(b0), "f"(b1));
}

template <int TN, typename AT, typename XT, typename St>
__device__ __forceinline__ void block_mm(const AT* __restrict__ A, int lda, const XT* __restrict__ X,
                                         int ldx, int R, int N, int K, int KS, St&& st) {
    const int nRT = R >> 2, nNT = N / TN;
    const int wn = tile_cols_wn<TN>(nNT);
    const int wr = 32 / wn;
    const int nRB = (nRT + wr - 1) / wr, nNB = (nNT + wn - 1) / wn;
    const int nblk = nRB * nNB;
    const int KL = (((K >> 2) + KS - 1) / KS) << 2;
    const int items = KS * nblk * 32;
    for (int it = threadIdx.x; it < items; it += blockDim.x) {
        const int lane = it & 31, wi = it >> 5;
        const int blk = wi % nblk, ks = wi / nblk;
        const int rt = (blk % nRB) * wr + lane % wr;
        const int nt = (blk / nRB) * wn + lane / wr;
        if (rt >= nRT || nt >= nNT) continue;
        const int k0 = ks * KL, k1 = min(K, k0 + KL);
        float acc[4][TN];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;
        const AT* ap = A + rt * 4;
        const XT* xp = X + nt * TN;
#pragma unroll 2
        for (int k = k0; k < k1; k += 4) {
            float a[4][4], x[4][TN];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                load4(ap + (size_t)(k + q) * lda, a[q]);
#pragma unroll
                for (int h = 0; h < TN; h += 4) {
                    float t4[4];
                    load4(xp + (size_t)(k + q) * ldx + h, t4);
#pragma unroll
                    for (int e = 0; e < 4; ++e) x[q][h + e] = t4[e];
                }
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < TN; j += 2) ffma2(acc[i][j], acc[i][j + 1], a[q][i], x[q][j], x[q][j + 1]);
        }
        st(ks, rt * 4, nt * TN, acc);
    }
}

template <typename T> struct Vec4;
template <> struct Vec4<float> {
    typedef float4 type;
    static __device__ __forceinline__ float4 zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
};
template <> struct Vec4<bf16> {
    typedef uint2 type;
    static __device__ __forceinline__ uint2 zero() { return make_uint2(0u, 0u); }
};

// dst[r*ncols + c] = src[r*ld + c] for r < nrv, c < ncv, zero elsewhere in the
// nrows x ncols tile.  L1 is bypassed (rows are written by other blocks during
// the kernel); 8 loads per thread are in flight before their stores.
template <typename T>
__device__ __forceinline__ void copy_tile(T* __restrict__ dst, int nrows, int ncols,
                                          const T* __restrict__ src, size_t ld, int nrv, int ncv) {
    constexpr int UN = 8;
    const int tid = threadIdx.x, nth = blockDim.x;
    const bool vec = (ncols & 3) == 0 && ncv == ncols && (ld & 3) == 0 &&
                     (reinterpret_cast<uintptr_t>(src) & (4 * sizeof(T) - 1)) == 0;
    if (vec) {
        typedef typename Vec4<T>::type V;
        const int cv = ncols >> 2;
        const int total = nrows * cv;
        for (int base = tid; base < total; base += nth * UN) {
            V v[UN];
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                v[u] = Vec4<T>::zero();
                if (i < total && i / cv < nrv)
                    v[u] = __ldcg(reinterpret_cast<const V*>(src + (size_t)(i / cv) * ld) + i % cv);
            }
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                if (i < total) reinterpret_cast<V*>(dst)[i] = v[u];
            }
        }
    } else {
        const int total = nrows * ncols;
        for (int base = tid; base < total; base += nth * UN) {
            T v[UN];
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                v[u] = from_f<T>(0.f);
                const int r = i / ncols, c = i % ncols;
                if (i < total && r < nrv && c < ncv) v[u] = ld_cg(src + (size_t)r * ld + c);
            }
#pragma unroll
            for (int u = 0; u < UN; ++u) {
                const int i = base + u * nth;
                if (i < total) dst[i] = v[u];
            }
        }
    }
}

constexpr int kRecThreads = 256;   // threads per recurrent block

// Column-tile width of the block_mm calls on an N-column operand.
__host__ __device__ constexpr int rec_tn(int N) { return N % 8 == 0 ? 8 : 4; }

// Row stride of the backward's gate-derivative tile (Bs columns): the
// padding spreads the unit-fastest stores of its gate-major rows over banks.
__host__ __device__ constexpr int bwd_lda(int Bs) { return Bs + 4; }

inline int pick_ks(int R, int N, int K) {
    const int nT = (R / 4) * (N / rec_tn(N));
    int ks = 1;
    while (nT * ks * 2 <= kRecThreads && K / (ks * 2) >= 16) ks *= 2;
    return ks;
}

// ============================================================== forward
template <typename WT>
__global__ void __launch_bounds__(kRecThreads, 1) fwd_rec_kernel(FwdRecArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const RecPlan& p = a.p;
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int Hp = (H + 3) & ~3;
    const int U = p.U, R = 4 * U, Bs = p.Bs, KS = p.KS;
    WT* Ws = reinterpret_cast<WT*>(smem);                              // [Hp][R]
    size_t off = align16((size_t)Hp * R * sizeof(WT));
    WT* hs = reinterpret_cast<WT*>(smem + off);                        // [Hp][Bs]
    off += align16((size_t)Hp * Bs * sizeof(WT));
    // K-slice partial sums, column-major per slice so that a thread's 4-row
    // tile column is one 16-byte store and a unit's 4 gates one 16-byte load
    float* red = reinterpret_cast<float*>(smem + off);                 // [KS][Bs][R]
    off += align16((size_t)KS * R * Bs * sizeof(float));
    float* cs = reinterpret_cast<float*>(smem + off);                  // [Bg][U]
    off += align16((size_t)U * p.Bg * sizeof(float));
    uint64_t* hbar = reinterpret_cast<uint64_t*>(smem + ((off + 7) & ~size_t(7)));

    const int j = blockIdx.x % p.nu;
    const int bg = (blockIdx.x / p.nu) % p.nbg;
    const int d = blockIdx.x / (p.nu * p.nbg);
    const int u0 = j * U, nU = min(U, H - u0);
    const int b0 = bg * p.Bg, nB = min(p.Bg, B - b0);
    const WT* h0 = static_cast<const WT*>(a.h0);
    WT* hT = static_cast<WT*>(a.hT);
    WT* hseq = static_cast<WT*>(a.hseq);
    WT* out = static_cast<WT*>(a.out);
    WT* h_n = static_cast<WT*>(a.h_n);
    const int tid = threadIdx.x, nth = blockDim.x;

    {
        typedef typename Vec4<WT>::type V;
        const V* s4 = reinterpret_cast<const V*>(static_cast<const WT*>(a.wpk) +
                                                 ((size_t)d * p.nu + j) * Hp * R);
        V* d4 = reinterpret_cast<V*>(Ws);
        for (int i = tid; i < Hp * R / 4; i += nth) d4[i] = s4[i];
    }
    for (int i = tid; i < U * p.Bg; i += nth) {
        const int ul = i % U, bl = i / U;
        float c = 0.f;
        if (a.c0 && ul < nU && bl < nB) c = a.c0[((size_t)d * B + b0 + bl) * H + u0 + ul];
        cs[i] = c;
    }
    if (tid == 0) {
        tc::mbar_init(hbar, 1);
        tc::fence_mbar_init();
    }
    __syncthreads();
    if (nB <= 0) return;   // plans never leave a group empty

    unsigned* ctr = a.ctr + d * p.nbg + bg;
    const size_t ldseq = (size_t)D * H;
    const size_t tile = (size_t)H * p.Bg;                       // exchange elements per (t, group)
    WT* hT_grp = hT + (size_t)bg * tile;                        // + (d*T + t) * nbg * tile
    const size_t hT_tstride = (size_t)p.nbg * tile;
    // one bulk copy per step when the group's tile is the whole shared tile
    const bool bulk = Bs == p.Bg && Hp == H && ((tile * sizeof(WT)) & 15) == 0 &&
                      ((reinterpret_cast<uintptr_t>(hT) & 15) == 0);
    uint32_t hphase = 0;
    const int np0 = nU * min(Bs, nB);
    const bool tr0 = blockIdx.x == 0 && tid == 0;   // the traced thread
    auto store_red = [&](int ks, int r0, int n0, auto& acc) {
        constexpr int tn = sizeof(acc[0]) / sizeof(float);
        float* rp = red + ((size_t)ks * Bs + n0) * R + r0;
#pragma unroll
        for (int j = 0; j < tn; ++j)
            *reinterpret_cast<float4*>(rp + (size_t)j * R) = make_float4(acc[0][j], acc[1][j], acc[2][j], acc[3][j]);
    };
    for (int s = 0; s < T; ++s) {
        const int t = d == 0 ? s : T - 1 - s;
        const int tp = d == 0 ? t - 1 : t + 1;
        // Gx of this thread's first-sub-tile pairs does not depend on other
        // blocks: fetch it before waiting.  Pair i: unit ul = i % nU, row
        // bl = i / nU (units fastest: Gx, outputs and saved state of
        // consecutive threads are contiguous).
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
        trace_mark(a.trace, tr0, s, 0);
        if (s > 0 && p.nu > 1) {
            if (!block_wait_geq(ctr, (unsigned)(p.nu * s), a.status, a.timeout_ns)) return;
        }
        trace_mark(a.trace, tr0, s, 1);
        for (int bs0 = 0; bs0 < nB; bs0 += Bs) {
            const int nb = min(Bs, nB - bs0);
            if (s == 0) {
                for (int i = tid; i < Hp * Bs; i += nth) {
                    const int k = i / Bs, bl = i % Bs;
                    WT v = from_f<WT>(0.f);
                    if (h0 && k < H && bl < nb) v = h0[((size_t)d * B + b0 + bs0 + bl) * H + k];
                    hs[i] = v;
                }
            } else if (bulk) {
                if (tid == 0) {
                    // order the previous step's generic reads of hs and the
                    // other blocks' generic writes of hT before the async copy
                    tc::fence_proxy_async_smem();
                    tc::fence_proxy_async_global();
                    tc::mbar_arrive_expect_tx(hbar, (uint32_t)(tile * sizeof(WT)));
                    tc::bulk_load(hs, hT_grp + ((size_t)d * T + tp) * hT_tstride, (uint32_t)(tile * sizeof(WT)), hbar);
                }
                volatile int never = 0;
                if (!tc::mbar_wait(hbar, hphase, &never, a.status, a.timeout_ns)) {
                    // the copy may still be writing into this block's shared
                    // memory: let it land (bounded) before the block leaves
                    const uint64_t t0 = globaltimer_ns();
                    while (!tc::mbar_try_wait(hbar, hphase) && globaltimer_ns() - t0 < 100000000ull) {
                    }
                    return;
                }
                hphase ^= 1;
            } else {
                copy_tile(hs, Hp, Bs, hT_grp + ((size_t)d * T + tp) * hT_tstride + bs0, (size_t)p.Bg, H, nb);
            }
            __syncthreads();
            if (bs0 == 0) trace_mark(a.trace, tr0, s, 2);
            if (rec_tn(Bs) == 8)
                block_mm<8>(Ws, R, hs, Bs, R, Bs, Hp, KS, store_red);
            else
                block_mm<4>(Ws, R, hs, Bs, R, Bs, Hp, KS, store_red);
            __syncthreads();
            if (bs0 == 0) trace_mark(a.trace, tr0, s, 3);
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
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int ks = 0; ks < KS; ++ks) {
                    const float4 r4 = *reinterpret_cast<const float4*>(red + ((size_t)ks * Bs + bl) * R + 4 * ul);
                    acc.x += r4.x; acc.y += r4.y; acc.z += r4.z; acc.w += r4.w;
                }
                const float pre[4] = {gxv.x + acc.x, gxv.y + acc.y, gxv.z + acc.z, gxv.w + acc.w};
                float& cref = cs[(bs0 + bl) * U + ul];
                // Padding of a variable-length row: the state stays as it was
                // (h from the gathered tile), the user output is 0, and the
                // exchange and the saved sequence carry the frozen h.
                const bool valid = !a.len || t < a.len[b];
                float c = cref;
                WT hv;
                float4 gates = make_float4(0.f, 0.f, 0.f, 0.f);
                if (!valid) {
                    hv = hs[(size_t)u * Bs + bl];
                } else {
                    const float ig = sigmoidf_(pre[0]);
                    const float fg = sigmoidf_(pre[1]);
                    const float gg = tanhf(pre[2]);
                    const float og = sigmoidf_(pre[3]);
                    c = fg * cref + ig * gg;
                    cref = c;
                    hv = from_f<WT>(og * tanhf(c));
                    gates = make_float4(ig, fg, gg, og);
                }
                hT_grp[((size_t)d * T + t) * hT_tstride + (size_t)u * p.Bg + bs0 + bl] = hv;
                if (hseq) hseq[((size_t)t * B + b) * ldseq + (size_t)d * H + u] = hv;
                if (out)
                    out[(size_t)t * a.out_st + (size_t)b * a.out_sb + (size_t)d * H + u] = valid ? hv : from_f<WT>(0.f);
                if (a.act) {
                    *reinterpret_cast<float4*>(a.act + (((size_t)d * T + t) * B + b) * G + 4 * u) = gates;
                    a.cst[(((size_t)d * T + t) * B + b) * H + u] = c;
                }
                if (s == T - 1) {
                    h_n[((size_t)d * B + b) * H + u] = hv;
                    a.c_n[((size_t)d * B + b) * H + u] = c;
                }
            }
            __syncthreads();
        }
        trace_mark(a.trace, tr0, s, 4);
        if (p.nu > 1 && s + 1 < T) {
            if (bulk) tc::fence_proxy_async_global();   // h_t is read by bulk copies
            if ((int)blockIdx.x == a.skip_block && s == a.skip_step)
                __syncthreads();   // fault injection: this step's arrival is withheld
            else
                block_arrive(ctr);
        }
        trace_mark(a.trace, tr0, s, 5);
    }
}

// ============================================================== backward
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

// WT: type of the resident W_hh rows (the weights' own type; products and
// sums are float32 either way).
template <typename WT>
__global__ void __launch_bounds__(kRecThreads, 1) bwd_rec_kernel(BwdRecArgs a) {
    extern __shared__ __align__(16) unsigned char smem[];
    const RecPlan& p = a.p;
    const int H = a.H, B = a.B, T = a.T, D = a.D, G = 4 * H;
    const int Hp = (H + 3) & ~3;
    const int U = p.U, R4 = 4 * U, Bs = p.Bs, Bg = p.Bg, LdA = bwd_lda(Bs);
    // Gate rows are gate-major within the block (row g*U + ul is gate g of
    // unit j0 + ul), and per-(row, unit) state is unit-fastest, so the
    // gate-gradient threads (units fastest) touch contiguous words.
    WT* Wr = reinterpret_cast<WT*>(smem);                             // [4U][Hp]
    size_t off = align16((size_t)R4 * Hp * sizeof(WT));
    float* daT = reinterpret_cast<float*>(smem + off);                // [4U][LdA]
    off += align16((size_t)R4 * LdA * 4);
    float* dcs = reinterpret_cast<float*>(smem + off);                // [Bg][U]
    off += align16((size_t)U * Bg * 4);
    float* dhs = reinterpret_cast<float*>(smem + off);                // [Bg][U]
    off += align16((size_t)U * Bg * 4);
    float* dbacc = reinterpret_cast<float*>(smem + off);              // [4][Bg][U]
    off += align16((size_t)4 * U * Bg * 4);
    // dh that padding of a variable-length row hands on unchanged (h_t = h_{t-1})
    float* dpass = reinterpret_cast<float*>(smem + off);              // [Bg][U]
    off += align16((size_t)U * Bg * 4);
    float* gpart = reinterpret_cast<float*>(smem + off);              // [CG][Bg][U]

    const int j = blockIdx.x % p.nu;
    const int bg = (blockIdx.x / p.nu) % p.nbg;
    const int d = blockIdx.x / (p.nu * p.nbg);
    const int j0 = j * U, nU = min(U, H - j0);
    const int b0 = bg * Bg, nB = min(Bg, B - b0);
    const int tid = threadIdx.x, nth = blockDim.x;
    {
        const uint4* s4 = reinterpret_cast<const uint4*>(static_cast<const WT*>(a.wr) +
                                                         ((size_t)d * p.nu + j) * R4 * Hp);
        uint4* d4 = reinterpret_cast<uint4*>(Wr);
        const int n16 = (int)((size_t)R4 * Hp * sizeof(WT) / 16);
        for (int i = tid; i < n16; i += nth) d4[i] = s4[i];
    }
    for (int i = tid; i < U * Bg; i += nth) {
        const int ul = i % U, bl = i / U;
        float dc = 0.f, dh = 0.f;
        if (ul < nU && bl < nB) {
            const size_t sidx = ((size_t)d * B + b0 + bl) * H + j0 + ul;
            if (a.grad_cn) dc = a.grad_cn[sidx];
            if (a.grad_hn) dh = a.grad_hn[sidx];
        }
        dcs[i] = dc;
        dhs[i] = dh;
    }
    for (int i = tid; i < 4 * U * Bg; i += nth) dbacc[i] = 0.f;
    for (int i = tid; i < U * Bg; i += nth) dpass[i] = 0.f;
    __syncthreads();
    if (nB <= 0) return;

    unsigned* ctr = a.ctr + d * p.nbg + bg;
    const size_t ldg = (size_t)D * G;
    // partial dh buffers: P[buf][d][bg][c][Bg][Hp]
    auto Pblk = [&](int buf, int c) {
        return a.P + ((((size_t)buf * D + d) * p.nbg + bg) * p.nu + c) * (size_t)Bg * Hp;
    };
    // gather: dhs[bl][ul] = sum_c P[buf][c][bl][j0+ul] (fixed order over c)
    const int U4 = U >> 2;
    const int CG = std::max(1, nth / (U4 * Bg));   // as sized by plan_bwd_rec
    auto gather = [&](int buf) {
        for (int i = tid; i < CG * U4 * nB; i += nth) {
            const int ul4 = i % U4, bl = (i / U4) % nB, cg = i / (U4 * nB);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            constexpr int UN = 8;
            for (int c0 = cg; c0 < p.nu; c0 += CG * UN) {
                float4 v[UN];
#pragma unroll
                for (int u = 0; u < UN; ++u) {
                    const int c = c0 + u * CG;
                    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                    if (c < p.nu)
                        v[u] = __ldcg(reinterpret_cast<const float4*>(Pblk(buf, c) + (size_t)bl * Hp + j0) + ul4);
                }
#pragma unroll
                for (int u = 0; u < UN; ++u) {
                    sum.x += v[u].x; sum.y += v[u].y; sum.z += v[u].z; sum.w += v[u].w;
                }
            }
            *reinterpret_cast<float4*>(gpart + ((size_t)cg * Bg + bl) * U + 4 * ul4) = sum;
        }
        __syncthreads();
        for (int i = tid; i < U * nB; i += nth) {
            const int ul = i % U, bl = i / U;
            float s = 0.f;
            for (int cg = 0; cg < CG; ++cg) s += gpart[((size_t)cg * Bg + bl) * U + ul];
            dhs[bl * U + ul] = s + dpass[bl * U + ul];
        }
        __syncthreads();
    };

    const int nb0 = min(Bs, nB);
    const bool tr0 = blockIdx.x == 0 && tid == 0;   // the traced thread
    for (int s = 0; s < T; ++s) {
        const int t = d == 0 ? T - 1 - s : s;
        // inputs of this thread's first-sub-tile pairs (pair i: unit
        // ul = i % U, row bl = i / U), fetched before the wait
        BwdPre pre[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int i = tid + q * nth;
            const int ul = i % U, bl = i / U;
            if (ul < nU && bl < nb0) pre[q] = bwd_fetch(a, d, t, b0 + bl, j0 + ul);
        }
        trace_mark(a.trace, tr0, s, 0);
        if (s > 0) {
            if (p.nu > 1 && !block_wait_geq(ctr, (unsigned)(p.nu * s), a.status, a.timeout_ns)) return;
            trace_mark(a.trace, tr0, s, 1);
            gather((s - 1) & 1);
        }
        trace_mark(a.trace, tr0, s, 2);
        for (int bs0 = 0; bs0 < nB; bs0 += Bs) {
            const int nb = min(Bs, nB - bs0);
            for (int i = tid, q = 0; i < U * Bs; i += nth, ++q) {
                const int ul = i % U, bl = i / U;
                if (ul >= nU || bl >= nb) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) daT[(g * U + ul) * LdA + bl] = 0.f;
                    continue;
                }
                const int b = b0 + bs0 + bl, jj = j0 + ul;
                const int sb = (bs0 + bl) * U + ul;   // per-(row, unit) state index
                float* dgp = a.dG + ((size_t)t * B + b) * ldg + (size_t)d * G + jj;
                if (a.len && t >= a.len[b]) {
                    // padding of a variable-length row: the state was held, so
                    // no gate gradient; dc and dh pass on unchanged (the output
                    // there is constant 0: grad_out does not enter)
                    dpass[sb] = dhs[sb];
                    dgp[0] = 0.f; dgp[H] = 0.f; dgp[2 * H] = 0.f; dgp[3 * H] = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) daT[(g * U + ul) * LdA + bl] = 0.f;
                    continue;
                }
                dpass[sb] = 0.f;
                const BwdPre v = (bs0 == 0 && q < 2) ? pre[q] : bwd_fetch(a, d, t, b, jj);
                const float ig = v.act.x, fg = v.act.y, gg = v.act.z, og = v.act.w;
                float& dcref = dcs[sb];
                const float dh = v.dy + dhs[sb];
                const float th = tanhf(v.c);
                const float dc = dcref + dh * og * (1.f - th * th);
                const float da_i = dc * gg * ig * (1.f - ig);
                const float da_f = dc * v.cp * fg * (1.f - fg);
                const float da_g = dc * ig * (1.f - gg * gg);
                const float da_o = dh * th * og * (1.f - og);
                dcref = dc * fg;
                dgp[0] = da_i;
                dgp[H] = da_f;
                dgp[2 * H] = da_g;
                dgp[3 * H] = da_o;
                daT[(0 * U + ul) * LdA + bl] = da_i;
                daT[(1 * U + ul) * LdA + bl] = da_f;
                daT[(2 * U + ul) * LdA + bl] = da_g;
                daT[(3 * U + ul) * LdA + bl] = da_o;
                float* dba = dbacc + sb;
                dba[0] += da_i;
                dba[(size_t)U * Bg] += da_f;
                dba[(size_t)2 * U * Bg] += da_g;
                dba[(size_t)3 * U * Bg] += da_o;
            }
            __syncthreads();
            if (bs0 == 0) trace_mark(a.trace, tr0, s, 3);
            // partial dh_{t-1}[b][0..Hp) from this block's 4U gate rows
            float* Pw = Pblk(s & 1, j) + (size_t)bs0 * Hp;
            auto store_p = [&](int, int r0, int n0, auto& acc) {
                constexpr int tn = sizeof(acc[0]) / sizeof(float);
#pragma unroll
                for (int jn = 0; jn < tn; ++jn) {
                    if (n0 + jn < nb)
                        *reinterpret_cast<float4*>(Pw + (size_t)(n0 + jn) * Hp + r0) =
                            make_float4(acc[0][jn], acc[1][jn], acc[2][jn], acc[3][jn]);
                }
            };
            if (rec_tn(Bs) == 8)
                block_mm<8>(Wr, Hp, daT, LdA, Hp, Bs, R4, 1, store_p);
            else
                block_mm<4>(Wr, Hp, daT, LdA, Hp, Bs, R4, 1, store_p);
            __syncthreads();
        }
        trace_mark(a.trace, tr0, s, 4);
        if (p.nu > 1 && !((int)blockIdx.x == a.skip_block && s == a.skip_step)) block_arrive(ctr);
        else __syncthreads();   // one block per group, or fault injection (arrival withheld)
        trace_mark(a.trace, tr0, s, 5);
    }
    if (T > 0) {
        if (p.nu > 1 && !block_wait_geq(ctr, (unsigned)(p.nu * T), a.status, a.timeout_ns)) return;
        gather((T - 1) & 1);
    }
    for (int i = tid; i < nU * nB; i += nth) {
        const int ul = i % nU, bl = i / nU;
        const size_t sidx = ((size_t)d * B + b0 + bl) * H + j0 + ul;
        a.dh0[sidx] = dhs[bl * U + ul];
        a.dc0[sidx] = dcs[bl * U + ul];
    }
    // bias-gradient partial of this block: sum over its batch rows, fixed order
    for (int i = tid; i < 4 * nU; i += nth) {
        const int q = i / nU, ul = i % nU;
        const float* col = dbacc + (size_t)q * Bg * U + ul;
        float sum = 0.f;
        for (int bl = 0; bl < nB; ++bl) sum += col[(size_t)bl * U];
        a.dbpart[((size_t)d * p.nbg + bg) * G + (size_t)q * H + j0 + ul] = sum;
    }
}

// Backward weight rows: out[d][p][k] (p < nu*4U, k < Hp) = W_hh[g*H + u][k]
// with block j = p / 4U, g = (p % 4U) / U and u = j*U + p % U (gate-major
// within each block's 4U rows), zero outside the matrix.
template <typename T>
__global__ void pack_hh_rows_kernel(PackHhBwdArgs a) {
    const int Hp = (a.H + 3) & ~3;
    T* out = static_cast<T*>(a.out);
    const int Rt = 4 * a.U * a.nu;
    const long long total = (long long)a.D * Rt * Hp;
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
         e += (long long)gridDim.x * blockDim.x) {
        const int k = (int)(e % Hp);
        const long long r2 = e / Hp;
        const int pr = (int)(r2 % Rt), d = (int)(r2 / Rt);
        const int pl = pr % (4 * a.U);
        const int g = pl / a.U, u = (pr / (4 * a.U)) * a.U + pl % a.U;
        out[e] = (u < a.H && k < a.H) ? static_cast<const T*>(a.w[d])[((long long)g * a.H + u) * a.H + k]
                                      : from_f<T>(0.f);
    }
}

}  // namespace

// ================================================================ planning
namespace {

// Plans depend only on their arguments: computed once per argument set.
struct PlanKey {
    int kind, H, B, D, dt, sms;
    size_t smem;
    bool operator<(const PlanKey& o) const {
        return std::tie(kind, H, B, D, dt, sms, smem) < std::tie(o.kind, o.H, o.B, o.D, o.dt, o.sms, o.smem);
    }
};

template <typename F>
RecPlan cached_plan(const PlanKey& k, F&& compute) {
    static std::mutex mu;
    static std::map<PlanKey, RecPlan> cache;
    {
        std::lock_guard<std::mutex> lk(mu);
        auto it = cache.find(k);
        if (it != cache.end()) return it->second;
    }
    const RecPlan p = compute();
    std::lock_guard<std::mutex> lk(mu);
    if (cache.size() > 4096) cache.clear();
    cache[k] = p;
    return p;
}

RecPlan plan_fwd_rec_uncached(int H, int B, int D, DType dt, int num_sms, size_t smem_max);
RecPlan plan_bwd_rec_uncached(int H, int B, int D, DType wdt, int num_sms, size_t smem_max);

}  // namespace

RecPlan plan_fwd_rec(int H, int B, int D, DType dt, int num_sms, size_t smem_max) {
    return cached_plan(PlanKey{0, H, B, D, (int)dt, num_sms, smem_max},
                       [&] { return plan_fwd_rec_uncached(H, B, D, dt, num_sms, smem_max); });
}

RecPlan plan_bwd_rec(int H, int B, int D, DType wdt, int num_sms, size_t smem_max) {
    return cached_plan(PlanKey{1, H, B, D, (int)wdt, num_sms, smem_max},
                       [&] { return plan_bwd_rec_uncached(H, B, D, wdt, num_sms, smem_max); });
}

namespace {

// Unit slices are powers of two: the products' warp tiling rounds a block's
// row tiles up to its lane layout, so other widths (e.g. 14 units, which
// would fill all 148 SMs at H = 512) cost as much per step as the next power
// of two (measured on the 2-layer workload: matvec 3.23 us either way).
RecPlan plan_fwd_rec_uncached(int H, int B, int D, DType dt, int num_sms, size_t smem_max) {
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
            RecPlan pl{};
            bool ok = false;
            for (; Bs >= 4; Bs -= 4) {
                const int R = 4 * U;
                const int KS = pick_ks(R, Bs, Hp);
                const size_t smem = align16h((size_t)Hp * R * es) + align16h((size_t)Hp * Bs * es) +
                                    align16h((size_t)KS * R * Bs * 4) + align16h((size_t)U * Bg * 4) + 16;
                if (smem <= smem_max) {
                    pl = RecPlan{nbg, Bg, nu, U, Bs, KS, kRecThreads, smem, ctas};
                    ok = true;
                    break;
                }
            }
            if (!ok) continue;
            const int nsub = (Bg + pl.Bs - 1) / pl.Bs;
            // per-step time estimate in SM cycles: FFMA work at ~75% of the SM's
            // 128 lanes, the exchange read (L2 bytes per block), fixed per-sub-tile
            // latency, and the group synchronisation
            const double fma = 4.0 * U * nsub * pl.Bs * (double)Hp;
            const double l2 = (double)Hp * Bg * es;
            const double cost = fma / 96.0 + l2 / 64.0 + nsub * 1500.0 + (nu > 1 ? 2500.0 : 0.0) +
                                (double)ctas * 1e-3;
            if (cost < best_cost) {
                best_cost = cost;
                best = pl;
            }
        }
    }
    return best;
}

RecPlan plan_bwd_rec_uncached(int H, int B, int D, DType wdt, int num_sms, size_t smem_max) {
    const int Hp = (H + 3) & ~3;
    const size_t wes = dtype_size(wdt);
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
            int Bs = std::min(((Bg + 3) / 4) * 4, 64);
            RecPlan pl{};
            bool ok = false;
            for (; Bs >= 4; Bs -= 4) {
                const int CG = std::max(1, kRecThreads / ((U / 4) * std::min(Bg, kRecThreads)));
                const size_t smem = align16h((size_t)4 * U * Hp * wes) + align16h((size_t)4 * U * bwd_lda(Bs) * 4) +
                                    3 * align16h((size_t)U * Bg * 4) + align16h((size_t)4 * U * Bg * 4) +
                                    align16h((size_t)CG * U * Bg * 4);
                if (smem <= smem_max) {
                    pl = RecPlan{nbg, Bg, nu, U, Bs, 1, kRecThreads, smem, ctas};
                    ok = true;
                    break;
                }
            }
            if (!ok) continue;
            const int nsub = (Bg + pl.Bs - 1) / pl.Bs;
            const double fma = 4.0 * U * nsub * pl.Bs * (double)Hp;
            const double l2 = (double)nu * Bg * U * 4 + (double)Bg * Hp * 4;
            const double cost = fma / 96.0 + l2 / 64.0 + nsub * 1500.0 + (nu > 1 ? 2500.0 : 0.0) +
                                (double)ctas * 1e-3;
            if (cost < best_cost) {
                best_cost = cost;
                best = pl;
            }
        }
    }
    return best;
}

}  // namespace

// ================================================================ launchers
cudaError_t launch_fwd_rec(const FwdRecArgs& a, cudaStream_t s) {
    FwdRecArgs args = a;
    void* params[] = {&args};
    const void* fn = a.dt == DType::F32 ? reinterpret_cast<const void*>(&fwd_rec_kernel<float>)
                                        : reinterpret_cast<const void*>(&fwd_rec_kernel<bf16>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)a.p.smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchCooperativeKernel(fn, dim3(a.p.ctas), dim3(a.p.threads), params, a.p.smem, s);
}

cudaError_t launch_bwd_rec(const BwdRecArgs& a, cudaStream_t s) {
    BwdRecArgs args = a;
    void* params[] = {&args};
    const void* fn = a.wdt == DType::F32 ? reinterpret_cast<const void*>(&bwd_rec_kernel<float>)
                                         : reinterpret_cast<const void*>(&bwd_rec_kernel<bf16>);
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)a.p.smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchCooperativeKernel(fn, dim3(a.p.ctas), dim3(a.p.threads), params, a.p.smem, s);
}

cudaError_t launch_pack_hh_rows(const PackHhBwdArgs& a, cudaStream_t s) {
    const long long total = (long long)a.D * 4 * a.U * a.nu * ((a.H + 3) & ~3);
    const long long g = std::min<long long>(std::max<long long>((total + 255) / 256, 1), 148LL * 16);
    if (a.dt == DType::F32)
        pack_hh_rows_kernel<float><<<(int)g, 256, 0, s>>>(a);
    else
        pack_hh_rows_kernel<bf16><<<(int)g, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace lstm
