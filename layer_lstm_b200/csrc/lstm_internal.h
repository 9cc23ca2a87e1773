// Internal interface between the C-ABI/scheduler (lstm_abi.cu) and the
// kernel launchers.  Not installed; no torch types anywhere.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace lstm {

enum class DType : int { F32 = 0, BF16 = 1 };

// Per-step timeline of block 0 of a recurrent kernel (instrumentation):
// trace[s * kTraceEvents + e] = %globaltimer (ns) when event e of step s
// happened; a null trace pointer records nothing.
constexpr int kTraceSteps = 512;
constexpr int kTraceEvents = 16;

inline size_t dtype_size(DType t) { return t == DType::F32 ? 4 : 2; }

// ---------------------------------------------------------------- GEMM
// C[M x N] (+)= A[M x K] * B[K x N] (+ bias[n]), float32 accumulate.
// A(m,k) = A[m*sAm + k*sAk], B(k,n) = B[k*sBk + n*sBn]; one of each pair of
// strides must be 1.  The output row of m is m, or with remap_T > 0 the
// (b,t) -> (t,b) row map m = b*T + t -> t*B + b (remap_B = B), or with
// remap_T < 0 the inverse map m = t*B + b -> b*T + t (T = -remap_T).
struct GemmArgs {
    int M, N, K;
    const void* A; long long sAm, sAk; DType ta;
    const void* B; long long sBk, sBn; DType tb;
    void* C; long long ldc; DType tc;   // tc: F32 or BF16 output
    const float* bias;                  // [N] or null
    int accumulate;                     // 1: C += result (C must be F32)
    int remap_T, remap_B;
};
cudaError_t launch_gemm(const GemmArgs& g, cudaStream_t s);

// Tensor-core GEMM (tcgen05): C[M x N] = A[M x K] * B[N x K]^T (+ bias[n])
// with each operand K-major, or MN-major when a_mn / b_mn (row strides lda,
// ldb elements, 16-byte multiples).  F32 operands use 3xTF32, BF16 operands kind::f16; the
// accumulator is float32.  Output column n < n_split goes to
// C[row*ldc + n], n >= n_split to C1[row*ldc1 + n - n_split] (C1 null: all to
// C).  Row map as in GemmArgs.  splitk > 1 needs ws (splitk*M*N floats).
struct TcGemmArgs {
    int M, N, K;
    DType dt;
    const void* A; long long lda;
    const void* B; long long ldb;
    float* C; long long ldc;
    float* C1; long long ldc1; int n_split;
    const float* bias;
    int accumulate;
    int remap_T, remap_B;
    int splitk;                 // largest K split to consider (<= 1: none)
    float* ws;                  // scratch for split-K partial sums, or null
    long long ws_floats;        // its capacity
    int* status;
    uint64_t timeout_ns;
    int num_sms;                // persistent grid size (SMs of the device)
    int a_mn;                   // 1: A stored [K][M] (row stride lda), contiguous in m
    int b_mn;                   // 1: B stored [K][N] (row stride ldb), contiguous in n
    int pdl;                    // 1: launch as a programmatic dependent of the preceding kernel in
                                // the stream (it may start once that kernel's blocks signalled and
                                // ends only after it); the GEMM must not read what that kernel writes
};
bool tc_gemm_supported(const TcGemmArgs& g);
// *nlaunch (if given) = kernels launched: 2 when K was split (GEMM + reduction).
cudaError_t launch_tc_gemm(const TcGemmArgs& g, cudaStream_t s, int* nlaunch = nullptr);

// dst[c*ldd + m] = src(m, c) for m < M, c < C.  src and h0 are float32, or
// bf16 when src_bf16; dst is float32, or bf16 rounded to nearest even when
// dst_bf16.
//  mode 0: src(m, c) = src[row(m)*lds + c], row(m) = m, or with bt_remap the
//          time-major index m = t*B + b read from a batch-first (b*T + t) array.
//  mode 1: h_{t-1} of one direction in its own time order: for m = t*B + b,
//          src(m, c) = src[(ts*B + b)*lds + c] with ts = t-1 (dir 0) or t+1
//          (dir 1) when 0 <= ts < T, else h0[b*C + c] (zero if h0 is null).
struct TransposeArgs {
    int M, C, mode;
    const void* src; long long lds;
    int bt_remap, T, B, dir;
    const void* h0;
    void* dst; long long ldd;
    int dst_bf16, src_bf16;
};
cudaError_t launch_transpose(const TransposeArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- packing
// Gate-interleaved row order used inside the library: packed row p = 4u + q
// holds standard row q*H + u (q = 0..3 for i, f, g, o).
struct PackIhArgs {
    int H, in, D;
    const void* w[2];          // per direction (G, in), standard order
    const void* b_ih[2];       // per direction G or null
    const void* b_hh[2];
    DType dt;
    void* wp;                  // [D*G][in] packed, dtype dt
    float* bias_p;             // [D*G] packed b_ih + b_hh (zeros without bias)
};
cudaError_t launch_pack_ih(const PackIhArgs& a, cudaStream_t s);

// Forward recurrent weights: [D][nu][H][4U] (k-major slices), zero padded.
struct PackHhFwdArgs {
    int H, D, nu, U;
    const void* w[2];
    DType dt;
    void* out;
};
cudaError_t launch_pack_hh_fwd(const PackHhFwdArgs& a, cudaStream_t s);

// Backward recurrent weights (float32): [D][nu*4U][Hp]; row p = 4u + q holds
// W_hh[q*H + u][:], zero padded.
struct PackHhBwdArgs {
    int H, D, nu, U;
    DType dt;                   // type of w and out (kept: bf16 weights stay bf16)
    const void* w[2];
    void* out;
};
cudaError_t launch_pack_hh_rows(const PackHhBwdArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- recurrence
struct RecPlan {
    int nbg, Bg, nu, U, Bs, KS, threads;
    size_t smem;
    int ctas;
};

struct FwdRecArgs {
    int H, B, T, D;
    RecPlan p;
    DType dt;
    const float* gx;            // [T][B][D*G] packed per direction, biases included
    const void* wpk;            // PackHhFwd layout
    const void* h0;             // [D][B][H] or null
    const float* c0;            // [D][B][H] or null
    void* hT;                   // [D][T][nbg][H][Bg] exchange copy of h (group-major, k-major)
    void* hseq;                 // [T][B][D*H] layer output, time-major
    void* out; long long out_st, out_sb;   // user out (top layer) or null; element strides
    void* h_n; float* c_n;      // [D][B][H]
    float* act; float* cst;     // [D][T][B][G] packed / [D][T][B][H], or null
    unsigned* ctr;              // [D*nbg] arrival counters, zero on entry
    int* status;
    uint64_t timeout_ns;
    unsigned long long* trace;  // [kTraceSteps][kTraceEvents] or null
    const int* len;             // [B] valid steps per row, or null (all T)
    int skip_block, skip_step;  // fault injection: that block withholds that step's arrival (-1: none)
};
cudaError_t launch_fwd_rec(const FwdRecArgs& a, cudaStream_t s);
RecPlan plan_fwd_rec(int H, int B, int D, DType dt, int num_sms, size_t smem_max);

// Tensor-core forward recurrence (bf16; inference, and training with act/cst).  W_hh packed rows
// [D*4H][H] bf16 (order 4u+q); hx exchange [D][T+1][B][H] bf16 with slot 0 =
// h0 (or zeros) filled before the launch.
struct TcRecPlan {
    bool ok;
    int nbg, Bg, N, nu, KH, kc_smem, stages, ctas;   // ctas = 2 per (d, bg, unit slice)
    size_t smem;
};
TcRecPlan plan_tc_rec(int H, int B, int D, int num_sms, size_t smem_max);

struct TcRecArgs {
    int H, B, T, D;
    TcRecPlan p;
    const float* gx;
    const void* wpk;
    const float* c0;
    void* hx;
    void* hseq;
    void* out; long long out_st, out_sb;
    void* h_n; float* c_n;
    unsigned* ctr;              // [D][nbg] group counters, 32 words apart, zeroed
    int* status;
    uint64_t timeout_ns;
    unsigned long long* trace;  // [kTraceSteps][kTraceEvents] or null
    const int* len;             // [B] valid steps per row, or null (all T)
    float* act;                 // training: [D][T][B][4H] gate activations, or null (inference)
    float* cst;                 // training: [D][T][B][H] cell states
};
cudaError_t launch_tc_rec(const TcRecArgs& a, cudaStream_t s);

// Tensor-core forward recurrence for float32 (3xTF32: W_hh and h split into
// tf32 hi and lo parts, products hi*hi + hi*lo + lo*hi, float32 sums).
// Clusters of C = H/128 blocks per (direction, batch group, 128 packed gate
// rows) split K = H; each block owns N/C of the group's N batch columns.
struct TcRec32Plan {
    bool ok;
    int nbg, Bg, N, nsl, C, KP, ctas;   // nsl slices of 128 rows, K part KP = H / C
    size_t smem;
};
TcRec32Plan plan_tc_rec32(int H, int B, int D, int num_sms, size_t smem_max);

struct TcRec32Args {
    int H, B, T, D;
    TcRec32Plan p;
    const float* gx;            // [T][B][D*4H] packed rows 4u+q, biases included
    const float* wpk;           // [D*4H][H] W_hh packed rows 4u+q, float32, or null: read w
    const float* w[2];          // W_hh of each direction as given ([4H][H], rows q*H + u), 16-byte aligned
    const float* h0;            // [D][B][H] or null
    const float* c0;            // [D][B][H] or null
    float* hx;                  // exchange [D][T+1][B][2H]: tf32 hi | remainder of h (slot 0 = h0)
    float* hseq;                // [T][B][D*H] or null
    float* out; long long out_st, out_sb;   // user output of the last layer, or null
    float* h_n; float* c_n;     // [D][B][H]
    float* act; float* cst;     // training: gate activations [D][T][B][4H] and cell states, or null
    unsigned* ctr;              // [D][nbg] counters, 32 words apart, zeroed
    int* status;
    uint64_t timeout_ns;
    const int* len;             // [B] valid steps per row, or null (all T)
    unsigned long long* trace;  // [kTraceSteps][kTraceEvents] or null
    int skip_block, skip_step;  // fault injection: that block withholds that step's arrival (-1: none)
};
// Exchange slot 0 (hi | lo of h0, or zeros); precedes launch_tc_rec32.
cudaError_t launch_rec32_slot0(const TcRec32Args& a, cudaStream_t s);
// *nlaunch (if given) = recurrent kernels launched (1, or D per direction).
cudaError_t launch_tc_rec32(const TcRec32Args& a, cudaStream_t s, int* nlaunch = nullptr);

// Tensor-core BPTT recurrence for float32 problems (3xTF32): clusters of
// H/32 blocks per 128-unit slice split K = 4H in parts of 128 gates (H = 128,
// 256 or 512); the gate gradients are exchanged split tf32 part | remainder
// through a ring of `slots` slots.
struct TcBwd32Plan {
    bool ok;
    int nbg, Bg, N, nsl, Cl, ctas, slots;
    size_t smem;
};
TcBwd32Plan plan_tc_bwd32(int H, int B, int D, int num_sms, size_t smem_max);
struct TcBwd32Args {
    int H, B, T, D;
    TcBwd32Plan p;
    const float* w[2];          // W_hh of each direction as given, [4H][H] float32
    const float* act;           // [D][T][B][4H] saved gate activations (i, f, g, o per unit)
    const float* cst;           // [D][T][B][H] saved cell states
    const float* c0;            // [D][B][H] or null
    const float* dy; long long dy_st, dy_sb;   // gradient reaching the layer output
    const float* grad_hn;       // [D][B][H] or null
    const float* grad_cn;       // [D][B][H] or null
    float* dG;                  // [T][B][D*4H] gate gradients, standard row order
    float* dax;                 // exchange [D][slots][B][8H]
    float* dh0; float* dc0;     // [D][B][H]
    float* dbpart;              // [D][nbg][4H] bias-gradient partials
    unsigned* ctr;              // [D][nbg] counters, 32 words apart, zeroed
    int* status;
    uint64_t timeout_ns;
    const int* len;             // [B] valid steps per row, or null (all T)
    unsigned long long* trace;  // [kTraceSteps][kTraceEvents] or null
    int skip_block, skip_step;  // fault injection: that block withholds that iteration's arrival (-1: none)
};
// *nlaunch (if given) = kernels launched.
cudaError_t launch_tc_bwd32(const TcBwd32Args& a, cudaStream_t s, int* nlaunch = nullptr);

// Tensor-core BPTT recurrence (bf16 W_hh; float32 state and gate
// gradients; the gate gradients of each step exchanged in bf16).  Clusters of
// 8 blocks per (direction, batch group, 128-unit slice) split K = 4H.
struct TcBwdPlan {
    bool ok;
    int nbg, Bg, N, nsl, nch, ctas;   // nsl slices of 128 units, nch 64-gate chunks per block
    size_t smem;
};
TcBwdPlan plan_tc_bwd(int H, int B, int D, int num_sms, size_t smem_max);

struct TcBwdArgs {
    int H, B, T, D;
    TcBwdPlan p;
    const void* wT;             // [D][H][4H] bf16: row u, column 4u'+q holds W_hh[q*H + u'][u]
    const float* act;           // [D][T][B][4H] gate activations (i, f, g, o of unit u at 4u)
    const float* cst;           // [D][T][B][H] cell states
    const float* c0;            // [D][B][H] or null
    const float* dy; long long dy_st, dy_sb;   // dL/dh_t of this layer's output, element (t, b, d*H + u)
    const float* grad_hn;       // [D][B][H] or null
    const float* grad_cn;       // [D][B][H] or null
    void* dG;                   // [T][B][D*4H] gate gradients, standard row order q*H + u
    int dG_bf16;                // dG in bf16 (rounded to nearest even) rather than float32
    void* dax;                  // [D][T+1][B][4H] bf16 exchange of the gate gradients (order 4u+q)
    float* dh0; float* dc0;     // [D][B][H]
    float* dbpart;              // [D][nbg][4H] bias-gradient partial of each batch group
    unsigned* ctr;              // [D][nbg] group counters, 32 words apart, zeroed
    int* status;
    uint64_t timeout_ns;
    const int* len;             // [B] valid steps per row, or null (all T)
};
// *nlaunch (if given) = kernels launched: D when the directions run one after another.
cudaError_t launch_tc_bwd(const TcBwdArgs& a, cudaStream_t s, int* nlaunch = nullptr);

// out[d][u][4u'+q] = W_hh[d][q*H + u'][u] (bf16), the rows of W_hh^T in the
// packed gate order of the tensor-core BPTT recurrence.
struct PackWtArgs {
    int H, D;
    DType dt;                   // element type of w and out
    const void* w[2];           // W_hh of each direction, [4H][H]
    void* out;                  // [D][H][4H]: out[d][u][4u'+q] = W[d][q*H + u'][u]
};
cudaError_t launch_pack_wT(const PackWtArgs& a, cudaStream_t s);

struct BwdRecArgs {
    int H, B, T, D;
    RecPlan p;
    const void* wr;             // [D][nu*4U][Hp] W_hh rows, packed order 4u+q, type wdt
    DType wdt;
    const float* act;           // [D][T][B][G] packed
    const float* cst;           // [D][T][B][H]
    const float* c0;            // [D][B][H] or null
    const float* dy; long long dy_st, dy_sb;   // dy(t,b,col) = dy[t*st + b*sb + col]
    const float* grad_hn;       // [D][B][H] or null
    const float* grad_cn;       // [D][B][H] or null
    float* dG;                  // [T][B][D*G], standard row order per direction
    float* dh0; float* dc0;     // [D][B][H]
    float* dbpart;              // [D][nbg][G]
    float* P;                   // [2][D][nbg][nu][Bg][Hp] partial dh exchange
    unsigned* ctr;
    int* status;
    uint64_t timeout_ns;
    unsigned long long* trace;  // [kTraceSteps][kTraceEvents] or null
    const int* len;             // [B] valid steps per row, or null (all T)
    int skip_block, skip_step;  // fault injection: that block withholds that step's arrival (-1: none)
};
cudaError_t launch_bwd_rec(const BwdRecArgs& a, cudaStream_t s);
RecPlan plan_bwd_rec(int H, int B, int D, DType wdt, int num_sms, size_t smem_max);

// db[d][r] = sum over groups of dbpart[d][g][r] (fixed order), written to
// both db_ih[d] and db_hh[d].
struct DbArgs {
    int G, D, nbg;
    const float* dbpart;
    float* db_ih[2];
    float* db_hh[2];
};
cudaError_t launch_db_reduce(const DbArgs& a, cudaStream_t s);

// dst(t,b,:) = src(t,b,:) for a (rows x width) sequence with arbitrary
// (t,b) element strides; used to make time-major copies.
struct SeqCopyArgs {
    int T, B, W;
    const void* src; long long s_st, s_sb;
    void* dst; long long d_st, d_sb;
    DType dt;
};
cudaError_t launch_seq_copy(const SeqCopyArgs& a, cudaStream_t s);

// Inter-layer dropout: dst[e] = keep(e) ? src[e] * scale : 0 for e < n (src
// may equal dst), keep(e) = (w >> 11) >= thresh with w word e mod 4 of
// Philox4x64-10 at key (seed, layer), counter (e / 4, 0, 0, 0).
struct DropoutArgs {
    long long n;
    const void* src; void* dst; DType dt;
    unsigned long long seed; int layer;
    unsigned long long thresh;   // ceil(p * 2^53)
    float scale;                 // 1 / (1 - p)
};
cudaError_t launch_dropout(const DropoutArgs& a, cudaStream_t s);

// dst[i] = src[i] for i < n, converting between float and bf16 (nearest even).
cudaError_t launch_convert(const void* src, DType st, void* dst, DType dt, long long n, cudaStream_t s);

}  // namespace lstm
