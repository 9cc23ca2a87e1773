// C-ABI entry points and host-side scheduler of the LSTM library.
//
// The forward follows the lstm.input contract of "Complete Trace: nn.LSTM"
// (Step 3): input, hx, params, has_biases, num_layers, bidirectional,
// batch_first -> output, h_n, c_n, with the shapes of the warp_nn
// "Long Short-Term Memory (LSTM)" page.  Per layer: a time-batched input
// projection Gx = X W_ih^T + b_ih + b_hh for both directions at once, then one
// persistent recurrent launch in which the directions run concurrently.  The
// backward runs the layers top-down: the persistent BPTT launch (data phase),
// then time-batched GEMMs for dW_ih, dW_hh and the layer-input gradient
// (weight phase), mirroring the data/weight split described under cuDNN
// Backward on the same page.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <cmath>
#include <vector>

#include "../../include/lstm.h"
#include "lstm_internal.h"

namespace lstm {
namespace {

struct DevInfo {
    int sms = 0;
    size_t smem_optin = 0;
    bool ok = false;
};

DevInfo device_info() {
    static std::mutex mu;
    static std::vector<DevInfo> cache;
    int dev = 0;
    DevInfo bad;
    if (cudaGetDevice(&dev) != cudaSuccess) return bad;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)cache.size() <= dev) cache.resize(dev + 1);
    if (!cache[dev].ok) {
        cudaDeviceProp prop;
        if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return bad;
        cache[dev].sms = prop.multiProcessorCount;
        cache[dev].smem_optin = prop.sharedMemPerBlockOptin;
        cache[dev].ok = true;
    }
    return cache[dev];
}

// Fault injection for the tests of the bounded waits (off unless set):
// LSTM_B200_DEBUG_SKIP_ARRIVAL="fwd:<block>:<step>" or "bwd:<block>:<step>"
// makes that block of every FFMA or float32 tensor-core forward (backward)
// recurrent launch withhold its arrival of that step, so the blocks of its group give up at their next
// counter wait (no copy is in flight there) and the call ends with
// LSTM_ERR_TIMEOUT in the status word.
struct SkipArrival {
    int fwd_block = -1, fwd_step = -1, bwd_block = -1, bwd_step = -1;
};

const SkipArrival& skip_arrival() {
    static SkipArrival v = [] {
        SkipArrival r;
        const char* e = getenv("LSTM_B200_DEBUG_SKIP_ARRIVAL");
        if (e && *e) {
            char which[8] = {0};
            int blk = -1, st = -1;
            if (sscanf(e, "%3[a-z]:%d:%d", which, &blk, &st) == 3 && blk >= 0 && st >= 0) {
                if (strcmp(which, "fwd") == 0) { r.fwd_block = blk; r.fwd_step = st; }
                if (strcmp(which, "bwd") == 0) { r.bwd_block = blk; r.bwd_step = st; }
            }
        }
        return r;
    }();
    return v;
}

uint64_t timeout_ns() {
    static uint64_t v = [] {
        const char* e = getenv("LSTM_B200_WAIT_TIMEOUT_NS");
        if (e && *e) return (uint64_t)strtoull(e, nullptr, 10);
        return (uint64_t)2000000000ull;   // 2 s: far above any healthy step
    }();
    return v;
}

// ------------------------------------------------------------ kernel timing
// When enabled, every kernel the library launches is bracketed by a pair of
// CUDA events on its stream; lstm_timing_read() resolves them into per-kind
// launch counts and summed device durations.
// Kind names carry the engine: _tc tensor cores (tcgen05), _ffma / _simt the
// CUDA cores.
enum Kind {
    K_PACK = 0, K_PROJ_TC, K_PROJ_SIMT, K_FWD_REC_TC, K_FWD_REC_FFMA, K_BWD_REC_FFMA, K_DW_TC, K_DW_SIMT,
    K_DX_TC, K_DX_SIMT, K_DB, K_COPY, K_TRANSPOSE, K_DROPOUT, K_BWD_REC_TC, K_COUNT
};
const char* const kKindNames[K_COUNT] = {"pack",       "proj_gemm_tc", "proj_gemm_simt", "fwd_rec_tc",
                                         "fwd_rec_ffma", "bwd_rec_ffma", "dw_gemm_tc",   "dw_gemm_simt",
                                         "dx_gemm_tc", "dx_gemm_simt", "db_reduce",    "seq_copy",
                                         "transpose",  "dropout", "bwd_rec_tc"};

// Dropout launch for boundary `layer` over n time-major elements.
DropoutArgs dropout_args(const lstm_desc* d, int layer, const void* src, void* dst, DType dt, long long n) {
    DropoutArgs a{};
    const double p = d->dropout;
    a.n = n; a.src = src; a.dst = dst; a.dt = dt;
    a.seed = d->dropout_seed; a.layer = layer;
    a.thresh = (unsigned long long)ceil(p * 9007199254740992.0);   // p * 2^53
    a.scale = (float)(1.0 / (1.0 - p));
    return a;
}

struct Timing {
    std::mutex mu;
    bool on = false;
    struct Pending { int kind; cudaEvent_t a, b; int n; };
    std::vector<Pending> pending;
    std::vector<cudaEvent_t> pool;
    double total_ms[K_COUNT] = {};
    long long launches[K_COUNT] = {};
};

Timing& timing() {
    static Timing t;
    return t;
}

cudaEvent_t take_event(Timing& tm) {
    cudaEvent_t e = nullptr;
    if (!tm.pool.empty()) {
        e = tm.pool.back();
        tm.pool.pop_back();
    } else if (cudaEventCreate(&e) != cudaSuccess) {
        e = nullptr;
    }
    return e;
}

// nlaunch: where f leaves the number of kernels it launched (null: one).
template <typename F>
cudaError_t timed(int kind, cudaStream_t s, F&& f, const int* nlaunch = nullptr) {
    Timing& tm = timing();
    if (!tm.on) return f();
    std::lock_guard<std::mutex> lk(tm.mu);
    cudaEvent_t a = take_event(tm), b = take_event(tm);
    if (!a || !b) return cudaErrorMemoryAllocation;
    cudaError_t e = cudaEventRecord(a, s);
    if (e != cudaSuccess) return e;
    e = f();
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(b, s);
    if (e != cudaSuccess) return e;
    tm.pending.push_back({kind, a, b, nlaunch ? *nlaunch : 1});
    return cudaSuccess;
}

// Launches of `kind` that ran inside another kind's timed interval (counted,
// their time is part of that interval).
void count_launches(int kind, int n) {
    Timing& tm = timing();
    if (!tm.on) return;
    std::lock_guard<std::mutex> lk(tm.mu);
    tm.launches[kind] += n;
}

// GEMM engine: tensor cores where the operands meet TMA's alignment rules,
// the CUDA-core kernel otherwise.  LSTM_B200_GEMM=simt forces the CUDA-core
// kernel everywhere (used by the tests to cover both engines).
bool tc_gemm_enabled() {
    static const bool v = [] {
        const char* e = getenv("LSTM_B200_GEMM");
        return !(e && strcmp(e, "simt") == 0);
    }();
    return v;
}

// Recurrence engine for bf16 inference: tensor cores when the plan fits,
// otherwise the CUDA-core kernel.  LSTM_B200_REC=simt forces the latter.
bool tc_rec_enabled() {
    static const bool v = [] {
        const char* e = getenv("LSTM_B200_REC");
        return !(e && strcmp(e, "simt") == 0);
    }();
    return v;
}

// Layer wavefront of the forward ("LSTM Forward Computation", Stack Multiple
// RNN Cells: layer k+1 consumes the h sequence layer k produces), for
// unidirectional stacks on the CUDA-core recurrence: the sequence is cut
// into chunks, layer k runs chunk c on its own stream while layer k+1 runs
// chunk c-1.  LSTM_B200_WAVEFRONT=1 turns it on, =0 off; unset: off.
bool wavefront_enabled() {
    static const bool v = [] {
        const char* e = getenv("LSTM_B200_WAVEFRONT");
        return e && strcmp(e, "1") == 0;
    }();
    return v;
}

// Steps per wavefront chunk (at least 2, so that inside one launch every
// block of a group has read the chunk's initial state before any block
// writes the final state the next chunk starts from).
int wavefront_chunk(int T) {
    static const int v = [] {
        const char* e = getenv("LSTM_B200_WAVEFRONT_CHUNK");
        return e && *e ? atoi(e) : 16;
    }();
    return std::max(2, std::min(v, T));
}

// Non-blocking streams of the layer wavefront, created on first use per
// device and kept for the life of the process.
constexpr int kAuxStreams = 3;

cudaStream_t aux_stream(int i) {
    static std::mutex mu;
    static std::vector<std::vector<cudaStream_t>> pool;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if ((int)pool.size() <= dev) pool.resize(dev + 1);
    if (pool[dev].empty()) {
        for (int k = 0; k < kAuxStreams; ++k) {
            cudaStream_t s = nullptr;
            if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
            pool[dev].push_back(s);
        }
    }
    return pool[dev][i % kAuxStreams];
}

constexpr size_t kAlign = 256;
inline size_t al(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Shapes and the planned kernel partitions for one description.  The plans
// depend on the device (SM count, shared memory), so the layout is computed
// for the current device.
struct Layout {
    int L, D, I, H, B, T, G;
    DType dt;
    size_t es;
    RecPlan fwd, bwd;
    TcRecPlan tcr;
    int nbg_ctr;       // counter stride per (layer, direction) of the FFMA forward recurrence
    bool bwd_ok;
    // workspace offsets
    TcBwdPlan tcb;     // tensor-core BPTT recurrence (bf16), if it fits
    size_t ctr_tcb, dax, wT_tcb;
    TcRec32Plan tc32;  // tensor-core forward recurrence for float32 (3xTF32), if it fits
    size_t ctr_tc32, hx32;
    TcBwd32Plan tcb32; // tensor-core BPTT recurrence for float32 (3xTF32), if it fits
    size_t ctr_tcb32, dax32;
    size_t status, ctr_f, ctr_b, ctr_tc, ctr_end, wih[32], bias[32], whh_f, whh_b, gx, hT, seq[2], dG, dseq[2], xt,
        dbpart, P, dGT, bop, wcatT, hx, whh_tc, bias_dummy, gemm_ws, total;
    size_t gemm_ws_floats;
    // bf16 backward: float32 staging of what it reads and writes
    size_t s_x, s_h0, s_gout, s_ghn, s_hs[2], s_dx, s_dh0, s_wih[32];
    // reserve offsets
    size_t act[32], cst[32], hseq[32], rtotal;   // per layer: [D][T][B][G], [D][T][B][H], [T][B][D*H]
    size_t hdrop[32];   // layers 0..L-2 with dropout: the next layer's input, [T][B][D*H]
    float dropout;
    // layer wavefront (forward): plan on each layer's share of the SMs, a
    // second Gx buffer (layers alternate), per-layer exchange buffers and
    // counters sized for one chunk
    bool wf;
    int wf_chunk;
    RecPlan fwd_wf;
    size_t gx2, whh_wf, hTw[32], ctr_w, wf_end;
};

int in_size(const Layout& l, int layer) { return layer == 0 ? l.I : l.D * l.H; }

constexpr int kMaxSplitK = 4;   // K splits the weight-gradient GEMMs may use

bool valid_desc(const lstm_desc* d) {
    if (!d) return false;
    if (d->input_size < 1 || d->hidden_size < 1 || d->num_layers < 1) return false;
    if (d->num_layers > 32) return false;
    if (d->bidirectional != 0 && d->bidirectional != 1) return false;
    if (d->batch < 0 || d->seq_len < 0) return false;
    if (d->dtype != LSTM_F32 && d->dtype != LSTM_BF16) return false;
    if (!(d->dropout >= 0.f && d->dropout < 1.f)) return false;   // also rejects NaN
    // sizes addressed with 32-bit loop counters inside kernels
    const long long H = d->hidden_size, I = d->input_size;
    if (H > (1 << 16) || I > (1 << 20)) return false;
    return true;
}

bool make_layout(const lstm_desc* d, Layout& l) {
    if (!valid_desc(d)) return false;
    DevInfo dev = device_info();
    if (!dev.ok) {
        // No device: plan against a nominal B200 so sizes can still be queried.
        dev.sms = 148;
        dev.smem_optin = 232448;
    }
    l.L = d->num_layers;
    l.D = d->bidirectional ? 2 : 1;
    l.I = d->input_size;
    l.H = d->hidden_size;
    l.B = d->batch;
    l.T = d->seq_len;
    l.G = 4 * l.H;
    l.dt = d->dtype == LSTM_F32 ? DType::F32 : DType::BF16;
    l.es = dtype_size(l.dt);
    const size_t smem_max = dev.smem_optin - 1024;
    const int Bp = l.B > 0 ? l.B : 1;
    l.fwd = plan_fwd_rec(l.H, Bp, l.D, l.dt, dev.sms, smem_max);
    if (l.fwd.ctas == 0) return false;
    l.bwd = plan_bwd_rec(l.H, Bp, l.D, l.dt, dev.sms, smem_max);
    l.bwd_ok = l.bwd.ctas > 0;
    l.tcr = l.dt == DType::BF16 ? plan_tc_rec(l.H, Bp, l.D, dev.sms, smem_max) : TcRecPlan{};
    l.tcb = l.dt == DType::BF16 ? plan_tc_bwd(l.H, Bp, l.D, dev.sms, smem_max) : TcBwdPlan{};
    l.tc32 = l.dt == DType::F32 ? plan_tc_rec32(l.H, Bp, l.D, dev.sms, smem_max) : TcRec32Plan{};
    l.tcb32 = l.dt == DType::F32 ? plan_tc_bwd32(l.H, Bp, l.D, dev.sms, smem_max) : TcBwd32Plan{};
    const size_t TB = (size_t)l.T * l.B;
    size_t o = 0;
    l.status = o; o += al(sizeof(int));
    l.nbg_ctr = l.fwd.nbg;
    l.ctr_f = o; o += al(sizeof(unsigned) * (size_t)l.L * l.D * l.nbg_ctr);
    l.ctr_b = o; o += al(sizeof(unsigned) * (size_t)l.L * l.D * (l.bwd_ok ? l.bwd.nbg : 1));
    // tensor-core recurrence: one counter per (layer, direction, group), each
    // on its own 128-byte line
    l.ctr_tc = o; o += al(l.tcr.ok ? sizeof(unsigned) * 32 * (size_t)l.L * l.D * l.tcr.nbg : 0);
    l.ctr_tcb = o; o += al(l.tcb.ok ? sizeof(unsigned) * 32 * (size_t)l.L * l.D * l.tcb.nbg : 0);
    l.ctr_tc32 = o; o += al(l.tc32.ok ? sizeof(unsigned) * 32 * (size_t)l.L * l.D * l.tc32.nbg : 0);
    l.ctr_tcb32 = o; o += al(l.tcb32.ok ? sizeof(unsigned) * 32 * (size_t)l.L * l.D * l.tcb32.nbg : 0);
    l.ctr_end = o;
    for (int k = 0; k < l.L; ++k) {
        l.wih[k] = o; o += al((size_t)l.D * l.G * in_size(l, k) * l.es);
        l.bias[k] = o; o += al((size_t)l.D * l.G * 4);
    }
    l.whh_f = o; o += al((size_t)l.D * l.fwd.nu * ((l.H + 3) & ~3) * 4 * l.fwd.U * l.es);
    const size_t Hp = (size_t)((l.H + 3) & ~3);
    l.whh_b = o; o += al(l.bwd_ok ? (size_t)l.D * l.bwd.nu * 4 * l.bwd.U * Hp * l.es : 0);
    l.gx = o; o += al(TB * l.D * l.G * 4);
    l.hT = o; o += al((size_t)l.T * l.D * l.fwd.nbg * l.fwd.Bg * l.H * l.es);   // [D][T][nbg][H][Bg]
    l.seq[0] = o; o += al(TB * l.D * l.H * l.es);
    l.seq[1] = o; o += al(TB * l.D * l.H * l.es);
    l.wf = false;
    if (wavefront_enabled() && l.D == 1 && l.L >= 2 && l.T >= 2) {
        l.fwd_wf = plan_fwd_rec(l.H, Bp, 1, l.dt, dev.sms / 2, smem_max);
        if (l.fwd_wf.ctas > 0) {
            l.wf = true;
            l.wf_chunk = wavefront_chunk(l.T);
            const int maxc = l.wf_chunk + 1;   // a short last chunk joins the one before it
            l.gx2 = o; o += al(TB * l.G * 4);
            l.whh_wf = o; o += al((size_t)l.L * l.fwd_wf.nu * Hp * 4 * l.fwd_wf.U * l.es);
            for (int k = 0; k < l.L; ++k) {
                l.hTw[k] = o;
                o += al((size_t)(2 * maxc) * l.fwd_wf.nbg * l.fwd_wf.Bg * l.H * l.es);
            }
            l.ctr_w = o; o += al(sizeof(unsigned) * (size_t)l.L * l.fwd_wf.nbg);
        }
    }
    l.wf_end = o;
    l.hx = l.hx32 = l.whh_tc = l.bias_dummy = 0;
    if (l.tcr.ok || l.tc32.ok) {
        // exchange of h: bf16 [D][T+1][B][H], or float32 hi | lo [D][T+1][B][2H]
        if (l.tcr.ok) { l.hx = o; o += al((size_t)l.D * (l.T + 1) * l.B * l.H * 2); }
        if (l.tc32.ok) { l.hx32 = o; o += al((size_t)l.D * (l.T + 1) * l.B * 2 * l.H * 4); }
        l.whh_tc = o; o += al((size_t)l.D * l.G * l.H * l.es);
        l.bias_dummy = o; o += al((size_t)l.D * l.G * 4);
    }
    // backward (float32 arithmetic for both dtypes)
    const size_t maxin = (size_t)(l.I > l.D * l.H ? l.I : l.D * l.H);
    l.dG = o; o += al(TB * l.D * l.G * 4);
    l.dseq[0] = o; o += al(TB * maxin * 4);
    l.dseq[1] = o; o += al(TB * maxin * 4);
    l.xt = o; o += al(TB * l.I * 4);
    const int nbg_db = std::max({l.bwd_ok ? l.bwd.nbg : 1, l.tcb.ok ? l.tcb.nbg : 1, l.tcb32.ok ? l.tcb32.nbg : 1});
    l.dbpart = o; o += al((size_t)l.D * nbg_db * l.G * 4);
    // tensor-core BPTT: packed W_hh^T and the bf16 exchange of the gate gradients
    l.wT_tcb = o; o += al(l.tcb.ok ? (size_t)l.D * l.H * l.G * 2 : 0);
    l.dax = o; o += al(l.tcb.ok ? (size_t)l.D * (l.T + 1) * l.B * l.G * 2 : 0);
    // float32 tensor-core BPTT: the ring of split gate gradients
    l.dax32 = o; o += al(l.tcb32.ok ? (size_t)l.D * l.tcb32.slots * l.B * 2 * l.G * 4 : 0);
    l.P = o; o += al(l.bwd_ok ? (size_t)2 * l.D * l.bwd.nbg * l.bwd.nu * l.bwd.Bg * Hp * 4 : 0);
    l.dGT = o; o += al(TB * l.D * l.G * 4);
    l.bop = o; o += al((size_t)l.D * (maxin + l.H) * TB * 4);
    l.wcatT = o; o += al(maxin * l.D * l.G * 4);
    // split-K partial sums of the weight-gradient GEMMs (up to 4 splits)
    l.gemm_ws_floats = (size_t)kMaxSplitK * l.G * (maxin + l.H);
    l.gemm_ws = o; o += al(l.gemm_ws_floats * 4);
    if (l.dt == DType::BF16) {
        const size_t states = (size_t)l.L * l.D * l.B * l.H;
        l.s_x = o; o += al(TB * l.I * 4);
        l.s_h0 = o; o += al(states * 4);
        l.s_gout = o; o += al(TB * l.D * l.H * 4);
        l.s_ghn = o; o += al(states * 4);
        l.s_hs[0] = o; o += al(TB * l.D * l.H * 4);
        l.s_hs[1] = o; o += al(TB * l.D * l.H * 4);
        l.s_dx = o; o += al(TB * l.I * 4);
        l.s_dh0 = o; o += al(states * 4);
        for (int k = 0; k < l.L; ++k) {
            l.s_wih[k] = o; o += al((size_t)l.D * l.G * in_size(l, k) * 4);
        }
    }
    l.total = o;
    size_t r = 0;
    for (int k = 0; k < l.L; ++k) {
        l.act[k] = r; r += al((size_t)l.D * TB * l.G * 4);
        l.cst[k] = r; r += al((size_t)l.D * TB * l.H * 4);
        l.hseq[k] = r; r += al(TB * l.D * l.H * l.es);
    }
    l.dropout = d->dropout;
    for (int k = 0; k < l.L; ++k) {
        const bool dropped = l.dropout > 0.f && k < l.L - 1;
        l.hdrop[k] = r; r += al(dropped ? TB * l.D * l.H * l.es : 0);
    }
    l.rtotal = r;
    return true;
}

inline char* P(void* base, size_t off) { return static_cast<char*>(base) + off; }

#define LSTM_CUDA(call)                                  \
    do {                                                 \
        if ((call) != cudaSuccess) return LSTM_ERR_CUDA; \
    } while (0)

}  // namespace

bool desc_is_valid(const lstm_desc* desc) { return valid_desc(desc); }

// Bytes at the start of the workspace that an inference forward
// (reserve == NULL) reads or writes: the status word, the counters, the
// packed weights, the projection output and the exchange / layer-output
// buffers all lie in front of the buffers only the backward uses.
// 0 for an invalid description.
size_t forward_workspace_prefix(const lstm_desc* desc) {
    Layout l;
    if (!make_layout(desc, l)) return 0;
    if (l.tcr.ok || l.tc32.ok) return l.bias_dummy + al((size_t)l.D * l.G * 4);
    return l.wf_end;
}

static_assert(kTraceSteps == LSTM_TRACE_MAX_STEPS && kTraceEvents == LSTM_TRACE_EVENTS,
              "trace buffer shape differs from the header");

// Per-step timeline of block 0 of the last traced recurrent launch
// (instrumentation, off unless lstm_trace_enable(1)).
__device__ unsigned long long g_trace[kTraceSteps * kTraceEvents];

struct TraceState {
    std::mutex mu;
    bool on = false;
    int kind = 0, steps = 0;   // last traced launch
};

TraceState& trace_state() {
    static TraceState t;
    return t;
}

// Trace buffer for a recurrent launch of `kind` (LSTM_TRACE_*) over `steps`
// steps, zeroed on the stream; null when tracing is off.
unsigned long long* trace_for(int kind, int steps, cudaStream_t s) {
    TraceState& ts = trace_state();
    std::lock_guard<std::mutex> lk(ts.mu);
    if (!ts.on) return nullptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_trace) != cudaSuccess) return nullptr;
    if (cudaMemsetAsync(p, 0, sizeof(unsigned long long) * kTraceSteps * kTraceEvents, s) != cudaSuccess)
        return nullptr;
    ts.kind = kind;
    ts.steps = std::min(steps, kTraceSteps);
    return static_cast<unsigned long long*>(p);
}

}  // namespace lstm

using namespace lstm;

extern "C" {

lstm_status lstm_trace_enable(int enable) {
    TraceState& ts = trace_state();
    std::lock_guard<std::mutex> lk(ts.mu);
    ts.on = enable != 0;
    return LSTM_OK;
}

int lstm_trace_read(unsigned long long* out, int max_steps, int* kind) {
    TraceState& ts = trace_state();
    std::lock_guard<std::mutex> lk(ts.mu);
    if (kind) *kind = ts.kind;
    if (!out || max_steps <= 0 || ts.kind == 0) return 0;
    const int n = std::min(max_steps, ts.steps);
    if (cudaMemcpyFromSymbol(out, g_trace, sizeof(unsigned long long) * (size_t)n * kTraceEvents) != cudaSuccess)
        return -1;
    return n;
}

size_t lstm_workspace_size(const lstm_desc* desc) {
    Layout l;
    if (!make_layout(desc, l)) return 0;
    return l.total;
}

size_t lstm_reserve_size(const lstm_desc* desc) {
    Layout l;
    if (!make_layout(desc, l)) return 0;
    return l.rtotal;
}

lstm_status lstm_timing_enable(int enable) {
    Timing& tm = timing();
    std::lock_guard<std::mutex> lk(tm.mu);
    tm.on = enable != 0;
    return LSTM_OK;
}

int lstm_timing_read(lstm_kernel_time* out, int max_entries) {
    Timing& tm = timing();
    std::lock_guard<std::mutex> lk(tm.mu);
    for (const auto& p : tm.pending) {
        float ms = 0.f;
        if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
            tm.total_ms[p.kind] += ms;
            tm.launches[p.kind] += p.n;
        } else {
            return -1;
        }
        tm.pool.push_back(p.a);
        tm.pool.push_back(p.b);
    }
    tm.pending.clear();
    int n = 0;
    for (int k = 0; k < K_COUNT && n < max_entries; ++k, ++n) {
        if (!out) break;
        out[n].name = kKindNames[k];
        out[n].launches = tm.launches[k];
        out[n].total_ms = tm.total_ms[k];
    }
    return out ? n : (int)K_COUNT;
}

void lstm_timing_reset(void) {
    Timing& tm = timing();
    std::lock_guard<std::mutex> lk(tm.mu);
    for (const auto& p : tm.pending) {
        cudaEventSynchronize(p.b);
        tm.pool.push_back(p.a);
        tm.pool.push_back(p.b);
    }
    tm.pending.clear();
    for (int k = 0; k < K_COUNT; ++k) {
        tm.total_ms[k] = 0.0;
        tm.launches[k] = 0;
    }
}

const char* lstm_status_string(lstm_status s) {
    switch (s) {
        case LSTM_OK: return "LSTM_OK";
        case LSTM_ERR_INVALID_ARG: return "LSTM_ERR_INVALID_ARG";
        case LSTM_ERR_UNSUPPORTED: return "LSTM_ERR_UNSUPPORTED";
        case LSTM_ERR_WORKSPACE: return "LSTM_ERR_WORKSPACE";
        case LSTM_ERR_CUDA: return "LSTM_ERR_CUDA";
        case LSTM_ERR_TIMEOUT: return "LSTM_ERR_TIMEOUT";
    }
    return "LSTM_ERR_UNKNOWN";
}

lstm_status lstm_query_status(void* workspace, cudaStream_t stream) {
    if (!workspace) return LSTM_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LSTM_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LSTM_ERR_CUDA;
    return st == 0 ? LSTM_OK : (lstm_status)st;
}

lstm_status lstm_forward(const lstm_desc* desc, const void* x, const void* h0, const float* c0,
                         const void* const* w_ih, const void* const* w_hh,
                         const void* const* b_ih, const void* const* b_hh,
                         void* out, void* h_n, float* c_n,
                         void* workspace, size_t ws_bytes,
                         void* reserve, size_t rs_bytes, cudaStream_t stream) {
    return lstm_forward_varlen(desc, nullptr, x, h0, c0, w_ih, w_hh, b_ih, b_hh, out, h_n, c_n, workspace,
                               ws_bytes, reserve, rs_bytes, stream);
}

lstm_status lstm_forward_varlen(const lstm_desc* desc, const int* lengths, const void* x, const void* h0,
                                const float* c0, const void* const* w_ih, const void* const* w_hh,
                                const void* const* b_ih, const void* const* b_hh,
                                void* out, void* h_n, float* c_n,
                                void* workspace, size_t ws_bytes,
                                void* reserve, size_t rs_bytes, cudaStream_t stream) {
    if (!valid_desc(desc)) return LSTM_ERR_INVALID_ARG;
    if (!w_ih || !w_hh) return LSTM_ERR_INVALID_ARG;
    const int LD = desc->num_layers * (desc->bidirectional ? 2 : 1);
    for (int i = 0; i < LD; ++i) {
        if (!w_ih[i] || !w_hh[i]) return LSTM_ERR_INVALID_ARG;
        if (desc->bias && (!b_ih || !b_hh || !b_ih[i] || !b_hh[i])) return LSTM_ERR_INVALID_ARG;
    }
    const long long BT = (long long)desc->batch * desc->seq_len;
    if (BT > 0 && (!x || !out)) return LSTM_ERR_INVALID_ARG;
    if (desc->batch > 0 && (!h_n || !c_n)) return LSTM_ERR_INVALID_ARG;
    if (!workspace) return LSTM_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return LSTM_ERR_INVALID_ARG;
    if (reserve && reinterpret_cast<uintptr_t>(reserve) % 256 != 0) return LSTM_ERR_INVALID_ARG;
    Layout l;
    if (!make_layout(desc, l)) return LSTM_ERR_UNSUPPORTED;
    if (ws_bytes < l.total) return LSTM_ERR_WORKSPACE;
    if (reserve && rs_bytes < l.rtotal) return LSTM_ERR_WORKSPACE;
    if (!device_info().ok) return LSTM_ERR_CUDA;

    const int L = l.L, D = l.D, H = l.H, B = l.B, T = l.T, G = l.G;
    const size_t es = l.es;
    const size_t state_elems = (size_t)D * B * H;   // elements per layer slice
    LSTM_CUDA(cudaMemsetAsync(workspace, 0, l.ctr_end, stream));   // status word and all counters
    if (B == 0) return LSTM_OK;
    if (T == 0) {
        // no step runs: h_n = h0, c_n = c0 (zeros when absent)
        const size_t n = (size_t)L * state_elems;
        if (h0) LSTM_CUDA(cudaMemcpyAsync(h_n, h0, n * es, cudaMemcpyDeviceToDevice, stream));
        else LSTM_CUDA(cudaMemsetAsync(h_n, 0, n * es, stream));
        if (c0) LSTM_CUDA(cudaMemcpyAsync(c_n, c0, n * 4, cudaMemcpyDeviceToDevice, stream));
        else LSTM_CUDA(cudaMemsetAsync(c_n, 0, n * 4, stream));
        return LSTM_OK;
    }
    int* status = reinterpret_cast<int*>(P(workspace, l.status));
    for (int k = 0; k < L; ++k) {
        const int in = in_size(l, k);
        PackIhArgs pk{};
        pk.H = H; pk.in = in; pk.D = D; pk.dt = l.dt;
        for (int d = 0; d < D; ++d) {
            pk.w[d] = w_ih[k * D + d];
            pk.b_ih[d] = desc->bias ? b_ih[k * D + d] : nullptr;
            pk.b_hh[d] = desc->bias ? b_hh[k * D + d] : nullptr;
        }
        pk.wp = P(workspace, l.wih[k]);
        pk.bias_p = reinterpret_cast<float*>(P(workspace, l.bias[k]));
        LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_ih(pk, stream); }));
    }
    // Input projection of layer k over `rows` (batch, time) rows of layer_in
    // (time-major rows, or batch-first x of layer 0 when remap) into Gx rows
    // starting at gx_out; tensor cores where TMA can address the operands.
    auto project = [&](int k, const void* in_ptr, float* gx_out, long long rows, bool remap,
                       cudaStream_t st) -> cudaError_t {
        const int in = in_size(l, k);
        GemmArgs g{};
        g.M = (int)rows; g.N = D * G; g.K = in;
        g.A = in_ptr; g.ta = l.dt; g.sAm = in; g.sAk = 1;
        g.B = P(workspace, l.wih[k]); g.tb = l.dt; g.sBk = 1; g.sBn = in;
        g.C = gx_out; g.tc = DType::F32; g.ldc = (long long)D * G;
        g.bias = reinterpret_cast<const float*>(P(workspace, l.bias[k]));
        g.accumulate = 0;
        if (remap) { g.remap_T = T; g.remap_B = B; }
        TcGemmArgs tg{};
        tg.M = g.M; tg.N = g.N; tg.K = g.K; tg.dt = l.dt;
        tg.A = g.A; tg.lda = in; tg.B = g.B; tg.ldb = in;
        tg.C = gx_out; tg.ldc = g.ldc;
        tg.bias = g.bias; tg.remap_T = g.remap_T; tg.remap_B = g.remap_B;
        tg.status = status; tg.timeout_ns = timeout_ns(); tg.num_sms = device_info().sms;
        if (tc_gemm_enabled() && tc_gemm_supported(tg)) {
            int nl = 1;
            return timed(K_PROJ_TC, st, [&] { return launch_tc_gemm(tg, st, &nl); }, &nl);
        }
        return timed(K_PROJ_SIMT, st, [&] { return launch_gemm(g, st); });
    };

    const bool tc_path = (l.tcr.ok || l.tc32.ok) && tc_rec_enabled();
    if (l.wf && !lengths && !(reserve && l.dropout > 0.f) && !tc_path) {
        // ------------------------------------------------ layer wavefront
        // Layer k runs on stream k (the caller's stream for k = 0, a pool
        // stream otherwise).  Chunk c of layer k > 0 waits for chunk c of
        // layer k-1, projects that chunk of its input, and runs its
        // recurrence from the state chunk c-1 left in h_n / c_n, so layer k
        // works on chunk c while layer k-1 works on chunk c+1.
        const int C = l.wf_chunk;
        std::vector<int> t0s;
        for (int t0 = 0; t0 < T; t0 += C) t0s.push_back(t0);
        if (t0s.size() > 1 && T - t0s.back() < 2) t0s.pop_back();   // a 1-step tail joins the chunk before
        const int nch = (int)t0s.size();
        std::vector<cudaStream_t> sts(L, stream);
        for (int k = 1; k < L; ++k) {
            sts[k] = aux_stream((k - 1) % kAuxStreams);
            if (!sts[k]) return LSTM_ERR_CUDA;
        }
        // events: fork, then "layer k finished chunk c"
        std::vector<cudaEvent_t> ev((size_t)L * nch + 1, nullptr);
        auto cleanup = [&] {
            for (cudaEvent_t e : ev)
                if (e) cudaEventDestroy(e);
        };
        for (auto& e : ev) {
            if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
                e = nullptr;
                cleanup();
                return LSTM_ERR_CUDA;
            }
        }
        auto fail = [&] { cleanup(); return LSTM_ERR_CUDA; };
        // layer 0's projection of the whole sequence, on the caller's stream
        if (project(0, x, reinterpret_cast<float*>(P(workspace, l.gx)), (long long)B * T, desc->batch_first != 0,
                    stream) != cudaSuccess)
            return fail();
        if (cudaEventRecord(ev[(size_t)L * nch], stream) != cudaSuccess) return fail();
        for (int k = 1; k < L; ++k)
            if (cudaStreamWaitEvent(sts[k], ev[(size_t)L * nch], 0) != cudaSuccess) return fail();
        // packed W_hh of every layer (the layers run at the same time)
        const RecPlan& pw = l.fwd_wf;
        const size_t whh_layer = (size_t)pw.nu * ((H + 3) & ~3) * 4 * pw.U * es;
        for (int k = 0; k < L; ++k) {
            PackHhFwdArgs ph{};
            ph.H = H; ph.D = 1; ph.nu = pw.nu; ph.U = pw.U; ph.dt = l.dt;
            ph.w[0] = w_hh[k];
            ph.out = P(workspace, l.whh_wf) + (size_t)k * whh_layer;
            if (timed(K_PACK, sts[k], [&] { return launch_pack_hh_fwd(ph, sts[k]); }) != cudaSuccess) return fail();
        }
        // issue in wavefront order: at stage q, layer k handles chunk q - k
        for (int q = 0; q < nch + L - 1; ++q) {
            for (int k = 0; k < L; ++k) {
                const int c = q - k;
                if (c < 0 || c >= nch) continue;
                cudaStream_t st = sts[k];
                const int t0 = t0s[c], t1 = c + 1 < nch ? t0s[c + 1] : T, Tc = t1 - t0;
                float* gxk = reinterpret_cast<float*>(P(workspace, k % 2 == 0 ? l.gx : l.gx2));
                if (k > 0) {
                    if (cudaStreamWaitEvent(st, ev[(size_t)(k - 1) * nch + c], 0) != cudaSuccess) return fail();
                    const void* below = reserve ? (const void*)P(reserve, l.hseq[k - 1]) : (const void*)P(workspace, l.seq[(k - 1) & 1]);
                    if (project(k, static_cast<const char*>(below) + (size_t)t0 * B * H * es,
                                gxk + (size_t)t0 * B * G, (long long)B * Tc, false, st) != cudaSuccess)
                        return fail();
                }
                unsigned* ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_w)) + (size_t)k * pw.nbg;
                if (cudaMemsetAsync(ctr, 0, sizeof(unsigned) * pw.nbg, st) != cudaSuccess) return fail();
                FwdRecArgs f{};
                f.H = H; f.B = B; f.T = Tc; f.D = 1; f.p = pw; f.dt = l.dt;
                f.gx = gxk + (size_t)t0 * B * G;
                f.wpk = P(workspace, l.whh_wf) + (size_t)k * whh_layer;
                char* hn_k = static_cast<char*>(h_n) + (size_t)k * state_elems * es;
                float* cn_k = c_n + (size_t)k * state_elems;
                if (c == 0) {
                    f.h0 = h0 ? static_cast<const char*>(h0) + (size_t)k * state_elems * es : nullptr;
                    f.c0 = c0 ? c0 + (size_t)k * state_elems : nullptr;
                } else {
                    f.h0 = hn_k;   // the state chunk c-1 ended in
                    f.c0 = cn_k;
                }
                void* hseq = reserve ? P(reserve, l.hseq[k]) : P(workspace, l.seq[k & 1]);
                f.hseq = (k < L - 1 || reserve) ? static_cast<char*>(hseq) + (size_t)t0 * B * H * es : nullptr;
                f.hT = P(workspace, l.hTw[k]);
                if (k == L - 1) {
                    f.out_st = desc->batch_first ? (long long)H : (long long)B * H;
                    f.out_sb = desc->batch_first ? (long long)T * H : (long long)H;
                    f.out = static_cast<char*>(out) + (size_t)t0 * f.out_st * es;
                }
                f.h_n = hn_k;
                f.c_n = cn_k;
                if (reserve) {
                    f.act = reinterpret_cast<float*>(P(reserve, l.act[k])) + (size_t)t0 * B * G;
                    f.cst = reinterpret_cast<float*>(P(reserve, l.cst[k])) + (size_t)t0 * B * H;
                }
                f.ctr = ctr;
                f.status = status;
                f.timeout_ns = timeout_ns();
                f.skip_block = f.skip_step = -1;
                if (timed(K_FWD_REC_FFMA, st, [&] { return launch_fwd_rec(f, st); }) != cudaSuccess) return fail();
                if (cudaEventRecord(ev[(size_t)k * nch + c], st) != cudaSuccess) return fail();
            }
        }
        // join: the caller's stream waits for the last chunk of every layer
        for (int k = 1; k < L; ++k)
            if (cudaStreamWaitEvent(stream, ev[(size_t)k * nch + nch - 1], 0) != cudaSuccess) return fail();
        cleanup();
        return LSTM_OK;
    }

    const void* layer_in = x;
    for (int k = 0; k < L; ++k) {
        const int in = in_size(l, k);
        // time-batched input projection for both directions
        GemmArgs g{};
        g.M = B * T; g.N = D * G; g.K = in;
        g.A = layer_in; g.ta = l.dt; g.sAm = in; g.sAk = 1;
        g.B = P(workspace, l.wih[k]); g.tb = l.dt; g.sBk = 1; g.sBn = in;
        g.C = P(workspace, l.gx); g.tc = DType::F32; g.ldc = (long long)D * G;
        g.bias = reinterpret_cast<const float*>(P(workspace, l.bias[k]));
        g.accumulate = 0;
        if (k == 0 && desc->batch_first) { g.remap_T = T; g.remap_B = B; }
        TcGemmArgs tg{};
        tg.M = g.M; tg.N = g.N; tg.K = g.K; tg.dt = l.dt;
        tg.A = g.A; tg.lda = in; tg.B = g.B; tg.ldb = in;
        tg.C = static_cast<float*>(g.C); tg.ldc = g.ldc;
        tg.bias = g.bias; tg.remap_T = g.remap_T; tg.remap_B = g.remap_B;
        tg.status = status; tg.timeout_ns = timeout_ns(); tg.num_sms = device_info().sms;
        if (tc_gemm_enabled() && tc_gemm_supported(tg)) {
            int nl = 1;
            LSTM_CUDA(timed(K_PROJ_TC, stream, [&] { return launch_tc_gemm(tg, stream, &nl); }, &nl));
        } else {
            LSTM_CUDA(timed(K_PROJ_SIMT, stream, [&] { return launch_gemm(g, stream); }));
        }

        void* hseq_tc = reserve ? P(reserve, l.hseq[k]) : P(workspace, l.seq[k & 1]);
        if (tc_path && l.tc32.ok) {
            // float32 tensor-core recurrence (3xTF32): the kernel reads W_hh
            // as given (its gate-major rows are the order it keeps in tensor
            // memory) when every direction's pointer is 16-byte aligned, else a
            // packed copy; the launcher fills exchange slot 0 from h0
            TcRec32Args tr{};
            tr.H = H; tr.B = B; tr.T = T; tr.D = D; tr.p = l.tc32;
            tr.gx = reinterpret_cast<const float*>(P(workspace, l.gx));
            bool w_direct = true;
            for (int d = 0; d < D; ++d) {
                tr.w[d] = static_cast<const float*>(w_hh[k * D + d]);
                w_direct = w_direct && (reinterpret_cast<uintptr_t>(w_hh[k * D + d]) & 15) == 0;
            }
            if (!w_direct) {
                PackIhArgs pw{};
                pw.H = H; pw.in = H; pw.D = D; pw.dt = l.dt;
                for (int d = 0; d < D; ++d) pw.w[d] = w_hh[k * D + d];
                pw.wp = P(workspace, l.whh_tc);
                pw.bias_p = reinterpret_cast<float*>(P(workspace, l.bias_dummy));
                LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_ih(pw, stream); }));
                tr.wpk = reinterpret_cast<const float*>(P(workspace, l.whh_tc));
            }
            tr.h0 = h0 ? static_cast<const float*>(h0) + (size_t)k * state_elems : nullptr;
            tr.c0 = c0 ? c0 + (size_t)k * state_elems : nullptr;
            tr.hx = reinterpret_cast<float*>(P(workspace, l.hx32));
            tr.hseq = (k < L - 1 || reserve) ? static_cast<float*>(hseq_tc) : nullptr;
            if (k == L - 1) {
                tr.out = static_cast<float*>(out);
                tr.out_st = desc->batch_first ? (long long)D * H : (long long)B * D * H;
                tr.out_sb = desc->batch_first ? (long long)T * D * H : (long long)D * H;
            }
            tr.h_n = static_cast<float*>(h_n) + (size_t)k * state_elems;
            tr.c_n = c_n + (size_t)k * state_elems;
            if (reserve) {
                tr.act = reinterpret_cast<float*>(P(reserve, l.act[k]));
                tr.cst = reinterpret_cast<float*>(P(reserve, l.cst[k]));
            }
            tr.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_tc32)) + (size_t)k * D * l.tc32.nbg * 32;
            tr.status = status;
            tr.timeout_ns = timeout_ns();
            tr.len = lengths;
            tr.trace = trace_for(LSTM_TRACE_FWD_REC_TC32, T, stream);
            tr.skip_block = skip_arrival().fwd_block;
            tr.skip_step = skip_arrival().fwd_step;
            LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_rec32_slot0(tr, stream); }));
            int nl = 1;
            LSTM_CUDA(timed(K_FWD_REC_TC, stream, [&] { return launch_tc_rec32(tr, stream, &nl); }, &nl));
            layer_in = hseq_tc;
            if (reserve && l.dropout > 0.f && k < L - 1) {
                void* dropped = P(reserve, l.hdrop[k]);
                const DropoutArgs da = dropout_args(desc, k, hseq_tc, dropped, l.dt, (long long)B * T * D * H);
                LSTM_CUDA(timed(K_DROPOUT, stream, [&] { return launch_dropout(da, stream); }));
                layer_in = dropped;
            }
            continue;
        }
        if (tc_path) {
            // tensor-core recurrence: packed W_hh rows, h0 into exchange slot 0
            PackIhArgs pw{};
            pw.H = H; pw.in = H; pw.D = D; pw.dt = l.dt;
            for (int d = 0; d < D; ++d) pw.w[d] = w_hh[k * D + d];
            pw.wp = P(workspace, l.whh_tc);
            pw.bias_p = reinterpret_cast<float*>(P(workspace, l.bias_dummy));
            LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_ih(pw, stream); }));
            for (int d = 0; d < D; ++d) {
                char* slot0 = P(workspace, l.hx) + (size_t)d * (T + 1) * B * H * 2;
                if (h0)
                    LSTM_CUDA(cudaMemcpyAsync(slot0, static_cast<const char*>(h0) + ((size_t)k * D + d) * B * H * 2,
                                              (size_t)B * H * 2, cudaMemcpyDeviceToDevice, stream));
                else
                    LSTM_CUDA(cudaMemsetAsync(slot0, 0, (size_t)B * H * 2, stream));
            }
            TcRecArgs tr{};
            tr.H = H; tr.B = B; tr.T = T; tr.D = D; tr.p = l.tcr;
            tr.gx = reinterpret_cast<const float*>(P(workspace, l.gx));
            tr.wpk = P(workspace, l.whh_tc);
            tr.c0 = c0 ? c0 + (size_t)k * state_elems : nullptr;
            tr.hx = P(workspace, l.hx);
            tr.hseq = (k < L - 1 || reserve) ? hseq_tc : nullptr;
            if (k == L - 1) {
                tr.out = out;
                tr.out_st = desc->batch_first ? (long long)D * H : (long long)B * D * H;
                tr.out_sb = desc->batch_first ? (long long)T * D * H : (long long)D * H;
            }
            tr.h_n = static_cast<char*>(h_n) + (size_t)k * state_elems * es;
            tr.c_n = c_n + (size_t)k * state_elems;
            tr.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_tc)) + (size_t)k * D * l.tcr.nbg * 32;
            tr.status = status;
            tr.timeout_ns = timeout_ns();
            tr.trace = trace_for(LSTM_TRACE_FWD_REC_TC, T, stream);
            tr.len = lengths;
            if (reserve) {
                tr.act = reinterpret_cast<float*>(P(reserve, l.act[k]));
                tr.cst = reinterpret_cast<float*>(P(reserve, l.cst[k]));
            }
            LSTM_CUDA(timed(K_FWD_REC_TC, stream, [&] { return launch_tc_rec(tr, stream); }));
            layer_in = hseq_tc;
            if (reserve && l.dropout > 0.f && k < L - 1) {
                void* dropped = P(reserve, l.hdrop[k]);
                const DropoutArgs da = dropout_args(desc, k, hseq_tc, dropped, l.dt, (long long)B * T * D * H);
                LSTM_CUDA(timed(K_DROPOUT, stream, [&] { return launch_dropout(da, stream); }));
                layer_in = dropped;
            }
            continue;
        }

        PackHhFwdArgs ph{};
        ph.H = H; ph.D = D; ph.nu = l.fwd.nu; ph.U = l.fwd.U; ph.dt = l.dt;
        for (int d = 0; d < D; ++d) ph.w[d] = w_hh[k * D + d];
        ph.out = P(workspace, l.whh_f);
        LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_hh_fwd(ph, stream); }));

        FwdRecArgs f{};
        f.H = H; f.B = B; f.T = T; f.D = D; f.p = l.fwd; f.dt = l.dt;
        f.gx = reinterpret_cast<const float*>(P(workspace, l.gx));
        f.wpk = P(workspace, l.whh_f);
        f.h0 = h0 ? static_cast<const char*>(h0) + (size_t)k * state_elems * es : nullptr;
        f.c0 = c0 ? c0 + (size_t)k * state_elems : nullptr;
        void* hseq = reserve ? P(reserve, l.hseq[k]) : P(workspace, l.seq[k & 1]);
        f.hseq = (k < L - 1 || reserve) ? hseq : nullptr;
        f.hT = P(workspace, l.hT);
        if (k == L - 1) {
            f.out = out;
            f.out_st = desc->batch_first ? (long long)D * H : (long long)B * D * H;
            f.out_sb = desc->batch_first ? (long long)T * D * H : (long long)D * H;
        }
        f.h_n = static_cast<char*>(h_n) + (size_t)k * state_elems * es;
        f.c_n = c_n + (size_t)k * state_elems;
        if (reserve) {
            f.act = reinterpret_cast<float*>(P(reserve, l.act[k]));
            f.cst = reinterpret_cast<float*>(P(reserve, l.cst[k]));
        }
        f.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_f)) + (size_t)k * D * l.nbg_ctr;
        f.status = status;
        f.timeout_ns = timeout_ns();
        f.trace = trace_for(LSTM_TRACE_FWD_REC_FFMA, T, stream);
        f.len = lengths;
        f.skip_block = skip_arrival().fwd_block;
        f.skip_step = skip_arrival().fwd_step;
        LSTM_CUDA(timed(K_FWD_REC_FFMA, stream, [&] { return launch_fwd_rec(f, stream); }));
        layer_in = hseq;
        if (reserve && l.dropout > 0.f && k < L - 1) {
            void* dropped = P(reserve, l.hdrop[k]);
            const DropoutArgs da = dropout_args(desc, k, hseq, dropped, l.dt, (long long)B * T * D * H);
            LSTM_CUDA(timed(K_DROPOUT, stream, [&] { return launch_dropout(da, stream); }));
            layer_in = dropped;
        }
    }
    return LSTM_OK;
}

lstm_status lstm_backward(const lstm_desc* desc, const void* x, const void* h0, const float* c0,
                          const void* const* w_ih, const void* const* w_hh,
                          const void* grad_out, const void* grad_hn, const float* grad_cn,
                          const void* reserve, size_t rs_bytes,
                          void* workspace, size_t ws_bytes,
                          void* dx, void* dh0, float* dc0,
                          float* const* dw_ih, float* const* dw_hh,
                          float* const* db_ih, float* const* db_hh, cudaStream_t stream) {
    return lstm_backward_varlen(desc, nullptr, x, h0, c0, w_ih, w_hh, grad_out, grad_hn, grad_cn, reserve,
                                rs_bytes, workspace, ws_bytes, dx, dh0, dc0, dw_ih, dw_hh, db_ih, db_hh, stream);
}

lstm_status lstm_backward_varlen(const lstm_desc* desc, const int* lengths, const void* x, const void* h0,
                                 const float* c0, const void* const* w_ih, const void* const* w_hh,
                                 const void* grad_out, const void* grad_hn, const float* grad_cn,
                                 const void* reserve, size_t rs_bytes,
                                 void* workspace, size_t ws_bytes,
                                 void* dx, void* dh0, float* dc0,
                                 float* const* dw_ih, float* const* dw_hh,
                                 float* const* db_ih, float* const* db_hh, cudaStream_t stream) {
    if (!valid_desc(desc)) return LSTM_ERR_INVALID_ARG;
    if (!w_ih || !w_hh || !dw_ih || !dw_hh) return LSTM_ERR_INVALID_ARG;
    const int LD = desc->num_layers * (desc->bidirectional ? 2 : 1);
    for (int i = 0; i < LD; ++i) {
        if (!w_ih[i] || !w_hh[i] || !dw_ih[i] || !dw_hh[i]) return LSTM_ERR_INVALID_ARG;
        if (desc->bias && (!db_ih || !db_hh || !db_ih[i] || !db_hh[i])) return LSTM_ERR_INVALID_ARG;
    }
    const long long BT = (long long)desc->batch * desc->seq_len;
    if (BT > 0 && (!x || !grad_out || !dx || !reserve)) return LSTM_ERR_INVALID_ARG;
    if (desc->batch > 0 && (!dh0 || !dc0)) return LSTM_ERR_INVALID_ARG;
    if (!workspace) return LSTM_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(workspace) % 256 != 0) return LSTM_ERR_INVALID_ARG;
    if (reserve && reinterpret_cast<uintptr_t>(reserve) % 256 != 0) return LSTM_ERR_INVALID_ARG;
    Layout l;
    if (!make_layout(desc, l)) return LSTM_ERR_UNSUPPORTED;
    if (!l.bwd_ok) return LSTM_ERR_UNSUPPORTED;
    if (ws_bytes < l.total) return LSTM_ERR_WORKSPACE;
    if (BT > 0 && rs_bytes < l.rtotal) return LSTM_ERR_WORKSPACE;
    if (!device_info().ok) return LSTM_ERR_CUDA;

    const int L = l.L, D = l.D, H = l.H, B = l.B, T = l.T, G = l.G;
    const size_t state = (size_t)D * B * H;
    LSTM_CUDA(cudaMemsetAsync(workspace, 0, l.ctr_end, stream));   // status word and all counters
    // weight gradients start from zero (T == 0 or B == 0 leave them zero)
    for (int k = 0; k < L; ++k) {
        for (int d = 0; d < D; ++d) {
            const int i = k * D + d;
            if (BT == 0) {
                LSTM_CUDA(cudaMemsetAsync(dw_ih[i], 0, (size_t)G * in_size(l, k) * 4, stream));
                LSTM_CUDA(cudaMemsetAsync(dw_hh[i], 0, (size_t)G * H * 4, stream));
                if (desc->bias) {
                    LSTM_CUDA(cudaMemsetAsync(db_ih[i], 0, (size_t)G * 4, stream));
                    LSTM_CUDA(cudaMemsetAsync(db_hh[i], 0, (size_t)G * 4, stream));
                }
            }
        }
    }
    if (B == 0) return LSTM_OK;
    if (T == 0) {
        const size_t n = (size_t)L * state;
        if (grad_hn) LSTM_CUDA(cudaMemcpyAsync(dh0, grad_hn, n * l.es, cudaMemcpyDeviceToDevice, stream));
        else LSTM_CUDA(cudaMemsetAsync(dh0, 0, n * l.es, stream));
        if (grad_cn) LSTM_CUDA(cudaMemcpyAsync(dc0, grad_cn, n * 4, cudaMemcpyDeviceToDevice, stream));
        else LSTM_CUDA(cudaMemsetAsync(dc0, 0, n * 4, stream));
        return LSTM_OK;
    }
    int* status = reinterpret_cast<int*>(P(workspace, l.status));
    float* dG = reinterpret_cast<float*>(P(workspace, l.dG));
    // Cell arithmetic, states and sums are float32.  A bf16 problem on the
    // tensor cores end to end (bfd) has the BPTT kernel store dG in bf16 and
    // the weight phase read its bf16 operands where they are (x, h0, W_ih,
    // the saved sequences); otherwise it reads float32 copies of its bf16
    // inputs.  grad_out and grad_hn enter the recurrence as float32 copies,
    // dx and dh0 leave through float32 staging.
    const bool bf = l.dt == DType::BF16;
    const long long BTl0 = (long long)B * T;
    // the tensor-core weight phase of layer k with operands of type wdt
    auto weight_phase_tc = [&](int k, DType wdt) {
        const int in = in_size(l, k);
        TcGemmArgs tw{};
        tw.M = G; tw.N = in + H; tw.K = (int)BTl0; tw.dt = wdt;
        tw.A = P(workspace, l.dGT); tw.lda = BTl0; tw.B = P(workspace, l.bop); tw.ldb = BTl0;
        TcGemmArgs tx{};
        tx.M = (int)BTl0; tx.N = in; tx.K = D * G; tx.dt = wdt;
        tx.A = dG; tx.lda = (long long)D * G; tx.B = P(workspace, l.wcatT); tx.ldb = (long long)D * G;
        return tc_gemm_enabled() && tc_gemm_supported(tw) && tc_gemm_supported(tx) &&
               (reinterpret_cast<uintptr_t>(dw_ih[k * D]) & 3) == 0;
    };
    bool bfd = bf && l.tcb.ok && tc_rec_enabled();
    for (int k = 0; k < L && bfd; ++k) bfd = weight_phase_tc(k, DType::BF16);
    auto stage = [&](const void* src, size_t off, size_t n) -> const float* {
        if (!src) return nullptr;
        if (!bf) return static_cast<const float*>(src);
        float* dst = reinterpret_cast<float*>(P(workspace, off));
        const cudaError_t e = launch_convert(src, DType::BF16, dst, DType::F32, (long long)n, stream);
        return e == cudaSuccess ? dst : nullptr;
    };
    const size_t BTs = (size_t)B * T;
    const float* xf = bfd ? nullptr : stage(x, l.s_x, BTs * l.I);
    const float* h0f = bfd ? nullptr : stage(h0, l.s_h0, (size_t)L * state);
    const float* goutf = stage(grad_out, l.s_gout, BTs * D * H);
    const float* ghnf = stage(grad_hn, l.s_ghn, (size_t)L * state);
    if ((!bfd && !xf) || !goutf || (h0 && !bfd && !h0f) || (grad_hn && !ghnf)) return LSTM_ERR_CUDA;
    std::vector<const float*> wihf(L * D);   // W_hh stays in its own type (resident rows)
    for (int k = 0; k < L && !bfd; ++k)
        for (int d = 0; d < D; ++d) {
            const int i = k * D + d;
            const size_t nih = (size_t)G * in_size(l, k);
            wihf[i] = stage(w_ih[i], bf ? l.s_wih[k] + (size_t)d * nih * 4 : 0, nih);
            if (!wihf[i]) return LSTM_ERR_CUDA;
        }
    // A sequence the forward saved in the reserve ([T][B][D*H]) as float32:
    // itself, or (bf16) its copy in staging slot `slot`.
    auto saved_seq = [&](size_t roff, int slot) -> const float* {
        const void* src = static_cast<const char*>(reserve) + roff;
        if (!bf) return static_cast<const float*>(src);
        float* dst = reinterpret_cast<float*>(P(workspace, l.s_hs[slot]));
        return launch_convert(src, DType::BF16, dst, DType::F32, (long long)(BTs * D * H), stream) == cudaSuccess
                   ? dst : nullptr;
    };
    const bool dropped = l.dropout > 0.f;   // layer k > 0 read the dropped output of layer k - 1
    float* dh0f = bf ? reinterpret_cast<float*>(P(workspace, l.s_dh0)) : static_cast<float*>(dh0);
    float* dxf = bf ? reinterpret_cast<float*>(P(workspace, l.s_dx)) : static_cast<float*>(dx);
    // time-major copy of x for the layer-0 weight gradient
    const float* x_tm = xf;
    // (bf16 end to end: x itself, time-major, for the MN-major weight phase)
    const void* x_tm_bf = bfd ? x : nullptr;
    if (desc->batch_first) {
        SeqCopyArgs sc{};
        sc.T = T; sc.B = B; sc.W = l.I; sc.dt = bfd ? DType::BF16 : DType::F32;
        sc.src = bfd ? x : static_cast<const void*>(xf); sc.s_st = l.I; sc.s_sb = (long long)T * l.I;
        sc.dst = P(workspace, l.xt); sc.d_st = (long long)B * l.I; sc.d_sb = l.I;
        LSTM_CUDA(timed(K_COPY, stream, [&] { return launch_seq_copy(sc, stream); }));
        if (bfd)
            x_tm_bf = P(workspace, l.xt);
        else
            x_tm = reinterpret_cast<const float*>(P(workspace, l.xt));
    }
    const float* dy = goutf;
    long long dy_st = desc->batch_first ? (long long)D * H : (long long)B * D * H;
    long long dy_sb = desc->batch_first ? (long long)T * D * H : (long long)D * H;
    int cur = 0;
    // float32: the weight-gradient GEMMs of layer k + 1 run beside layer k's
    // tensor-core BPTT recurrence, which leaves SMs idle (its operands are
    // copies the transposes made before; the recurrence writes none of them)
    const bool overlap_dw = !bf && l.tcb32.ok && tc_rec_enabled() && device_info().sms > l.tcb32.ctas;
    std::vector<TcGemmArgs> deferred_dw;
    for (int k = L - 1; k >= 0; --k) {
        const int in = in_size(l, k);
        // bf16: the tensor-core BPTT recurrence when its plan fits (the same
        // switch as the forward's engine), else the CUDA-core one
        const bool tcb = bf && l.tcb.ok && tc_rec_enabled();
        const bool tcb32 = !bf && l.tcb32.ok && tc_rec_enabled();
        if (!tcb && !tcb32) {
            PackHhBwdArgs pb{};
            pb.H = H; pb.D = D; pb.nu = l.bwd.nu; pb.U = l.bwd.U;
            pb.dt = l.dt;
            for (int d = 0; d < D; ++d) pb.w[d] = w_hh[k * D + d];
            pb.out = P(workspace, l.whh_b);
            LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_hh_rows(pb, stream); }));
        }

        BwdRecArgs b{};
        b.H = H; b.B = B; b.T = T; b.D = D; b.p = l.bwd;
        b.wr = P(workspace, l.whh_b);
        b.wdt = l.dt;
        b.P = reinterpret_cast<float*>(P(workspace, l.P));
        b.act = reinterpret_cast<const float*>(static_cast<const char*>(reserve) + l.act[k]);
        b.cst = reinterpret_cast<const float*>(static_cast<const char*>(reserve) + l.cst[k]);
        b.c0 = c0 ? c0 + (size_t)k * state : nullptr;
        b.dy = dy; b.dy_st = dy_st; b.dy_sb = dy_sb;
        b.grad_hn = ghnf ? ghnf + (size_t)k * state : nullptr;
        b.grad_cn = grad_cn ? grad_cn + (size_t)k * state : nullptr;
        b.dG = dG;
        b.dh0 = dh0f + (size_t)k * state;
        b.dc0 = dc0 + (size_t)k * state;
        b.dbpart = reinterpret_cast<float*>(P(workspace, l.dbpart));
        b.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_b)) + (size_t)k * D * l.bwd.nbg;
        b.status = status;
        b.timeout_ns = timeout_ns();
        b.trace = trace_for(LSTM_TRACE_BWD_REC_FFMA, T, stream);
        b.len = lengths;
        b.skip_block = skip_arrival().bwd_block;
        b.skip_step = skip_arrival().bwd_step;
        if (tcb) {
            PackWtArgs pw{};
            pw.H = H; pw.D = D; pw.dt = DType::BF16;
            for (int d = 0; d < D; ++d) pw.w[d] = w_hh[k * D + d];
            pw.out = P(workspace, l.wT_tcb);
            LSTM_CUDA(timed(K_PACK, stream, [&] { return launch_pack_wT(pw, stream); }));
            TcBwdArgs tb{};
            tb.H = H; tb.B = B; tb.T = T; tb.D = D; tb.p = l.tcb;
            tb.wT = pw.out;
            tb.act = b.act; tb.cst = b.cst; tb.c0 = b.c0;
            tb.dy = b.dy; tb.dy_st = b.dy_st; tb.dy_sb = b.dy_sb;
            tb.grad_hn = b.grad_hn; tb.grad_cn = b.grad_cn;
            tb.dG = dG;
            tb.dG_bf16 = bfd;
            tb.dax = P(workspace, l.dax);
            tb.dh0 = b.dh0; tb.dc0 = b.dc0; tb.dbpart = b.dbpart;
            tb.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_tcb)) + (size_t)k * D * l.tcb.nbg * 32;
            tb.status = status;
            tb.timeout_ns = timeout_ns();
            tb.len = lengths;
            int nl = 1;
            LSTM_CUDA(timed(K_BWD_REC_TC, stream, [&] { return launch_tc_bwd(tb, stream, &nl); }, &nl));
        } else if (tcb32) {
            TcBwd32Args tb{};
            tb.H = H; tb.B = B; tb.T = T; tb.D = D; tb.p = l.tcb32;
            for (int d = 0; d < D; ++d) tb.w[d] = static_cast<const float*>(w_hh[k * D + d]);   // read as given
            tb.act = b.act; tb.cst = b.cst; tb.c0 = b.c0;
            tb.dy = b.dy; tb.dy_st = b.dy_st; tb.dy_sb = b.dy_sb;
            tb.grad_hn = b.grad_hn; tb.grad_cn = b.grad_cn;
            tb.dG = dG;
            tb.dax = reinterpret_cast<float*>(P(workspace, l.dax32));
            tb.dh0 = b.dh0; tb.dc0 = b.dc0; tb.dbpart = b.dbpart;
            tb.ctr = reinterpret_cast<unsigned*>(P(workspace, l.ctr_tcb32)) + (size_t)k * D * l.tcb32.nbg * 32;
            tb.status = status;
            tb.timeout_ns = timeout_ns();
            tb.len = lengths;
            tb.trace = trace_for(LSTM_TRACE_BWD_REC_TC32, T, stream);
            tb.skip_block = skip_arrival().bwd_block;
            tb.skip_step = skip_arrival().bwd_step;
            int nl = 1, ndw = 0;
            LSTM_CUDA(timed(K_BWD_REC_TC, stream, [&] {
                cudaError_t e = launch_tc_bwd32(tb, stream, &nl);
                // the deferred GEMMs right behind it: the first as its programmatic
                // dependent on the SMs it leaves, the others in order after that one
                for (size_t i = 0; i < deferred_dw.size() && e == cudaSuccess; ++i) {
                    TcGemmArgs g = deferred_dw[i];
                    if (i == 0) {
                        g.pdl = 1;
                        g.num_sms = device_info().sms - l.tcb32.ctas;
                    }
                    int n = 1;
                    e = launch_tc_gemm(g, stream, &n);
                    ndw += n;
                }
                return e;
            }, &nl));
            count_launches(K_DW_TC, ndw);
            deferred_dw.clear();
        } else {
            LSTM_CUDA(timed(K_BWD_REC_FFMA, stream, [&] { return launch_bwd_rec(b, stream); }));
        }

        if (desc->bias) {
            DbArgs db{};
            db.G = G; db.D = D; db.nbg = tcb ? l.tcb.nbg : tcb32 ? l.tcb32.nbg : l.bwd.nbg; db.dbpart = b.dbpart;
            for (int d = 0; d < D; ++d) { db.db_ih[d] = db_ih[k * D + d]; db.db_hh[d] = db_hh[k * D + d]; }
            LSTM_CUDA(timed(K_DB, stream, [&] { return launch_db_reduce(db, stream); }));
        }
        // the layer's input and output sequences: bf16 where they are (bfd),
        // else float32 (copies)
        const float* layer_in = nullptr;
        const float* hs = nullptr;
        const void* lin_v;
        const void* hs_v;
        if (bfd) {
            lin_v = k == 0 ? x : static_cast<const char*>(reserve) + (dropped ? l.hdrop[k - 1] : l.hseq[k - 1]);
            hs_v = static_cast<const char*>(reserve) + l.hseq[k];
        } else {
            layer_in = k == 0 ? x_tm : saved_seq(dropped ? l.hdrop[k - 1] : l.hseq[k - 1], 1);
            hs = saved_seq(l.hseq[k], 0);
            if (!layer_in || !hs) return LSTM_ERR_CUDA;
            lin_v = k == 0 ? static_cast<const void*>(xf) : static_cast<const void*>(layer_in);
            hs_v = hs;
        }
        const size_t ses = bfd ? 2 : 4;   // element size of those sources
        const long long ldg = (long long)D * G, ldh = (long long)D * H;
        const long long BTl = (long long)B * T;
        float* din = k == 0 ? dxf : reinterpret_cast<float*>(P(workspace, l.dseq[cur]));
        // Tensor-core weight phase: dW = dG^T [In | H_prev] per direction over
        // K = B*T (one GEMM writes dW_ih and dW_hh), dIn = dG [W_ih_0; W_ih_1].
        // bf16 problems run it in bf16 (dG rounded to bf16, the other
        // operands exact in bf16, float32 accumulation), float32 problems in
        // 3xTF32.  The operand buffers hold either element type.
        const bool wbf = bf;
        const DType wdt = wbf ? DType::BF16 : DType::F32;
        const size_t wes = wbf ? 2 : 4;
        char* dGT = P(workspace, l.dGT);
        char* bop = P(workspace, l.bop);
        char* wcatT = P(workspace, l.wcatT);
        TcGemmArgs tw{};
        tw.M = G; tw.N = in + H; tw.K = (int)BTl; tw.dt = wdt;
        tw.A = dGT; tw.lda = BTl; tw.B = bop; tw.ldb = BTl;
        tw.C = dw_ih[k * D]; tw.ldc = in; tw.C1 = dw_hh[k * D]; tw.ldc1 = H; tw.n_split = in;
        tw.status = status; tw.timeout_ns = timeout_ns(); tw.num_sms = device_info().sms;
        tw.splitk = kMaxSplitK;
        tw.ws = reinterpret_cast<float*>(P(workspace, l.gemm_ws));
        tw.ws_floats = (long long)l.gemm_ws_floats;
        TcGemmArgs tx{};
        tx.M = (int)BTl; tx.N = in; tx.K = D * G; tx.dt = wdt;
        // bf16: dG itself (bfd) or a bf16 copy of it, written into dGT's space
        // once the dW GEMMs are done
        tx.A = (wbf && !bfd) ? static_cast<const void*>(dGT) : static_cast<const void*>(dG);
        tx.lda = ldg; tx.B = wcatT; tx.ldb = (long long)D * G;
        tx.C = din; tx.ldc = in;
        if (k == 0 && desc->batch_first) { tx.remap_T = -T; tx.remap_B = B; }
        tx.status = status; tx.timeout_ns = timeout_ns(); tx.num_sms = device_info().sms;
        const bool tc_ok = weight_phase_tc(k, wdt);
        // MN-major weight phase (bf16 end to end): dG, the time-major layer
        // input, the saved sequence and h0 are read where they are, dW_hh as a
        // GEMM over the shifted rows plus the h0 term (dX keeps its K-major W_ih
        // copy: one GEMM per direction reading W_ih MN-major took 0.58 ms on
        // c3's training shape against 0.32 + 0.06 for the copy and one GEMM).
        // float32 keeps the transposes: its MN-major operands take
        // the 128-byte swizzle on 32-byte granules, and the dW GEMMs of the
        // 2-layer H512 B64 step ran 0.74 ms that way against 0.44 ms K-major
        // (0.19 ms of transposes saved).
        const char* dG_v = reinterpret_cast<const char*>(dG);
        const void* lin_tm = k > 0 ? lin_v : bfd ? x_tm_bf : static_cast<const void*>(x_tm);
        const char* h0_v = bfd ? static_cast<const char*>(h0) : reinterpret_cast<const char*>(h0f);
        auto mn_gemm = [&](int d, int which) {   // which: 0 dW_ih, 1 dW_hh shifted, 2 h0 term
            TcGemmArgs g = tw;
            g.C1 = nullptr; g.ldc1 = 0; g.n_split = 0;
            g.a_mn = 1; g.b_mn = 1; g.lda = ldg;
            if (which == 0) {
                g.N = in; g.K = (int)BTl;
                g.A = dG_v + (size_t)d * G * wes;
                g.B = lin_tm; g.ldb = in;
                g.C = dw_ih[k * D + d]; g.ldc = in;
            } else if (which == 1) {
                g.N = H; g.K = (int)(BTl - B);
                g.A = dG_v + ((d == 0 ? (size_t)B * ldg : 0) + (size_t)d * G) * wes;          // rows t >= 1 / t <= T-2
                g.B = static_cast<const char*>(hs_v) + ((d == 0 ? 0 : (size_t)B * ldh) + (size_t)d * H) * wes;
                g.ldb = ldh;
                g.C = dw_hh[k * D + d]; g.ldc = H;
            } else {
                g.N = H; g.K = B;
                g.A = dG_v + ((d == 0 ? 0 : (size_t)(T - 1) * B * ldg) + (size_t)d * G) * wes;
                g.B = h0_v ? h0_v + ((size_t)k * D + d) * B * H * wes : nullptr; g.ldb = H;
                g.C = dw_hh[k * D + d]; g.ldc = H;
                g.accumulate = T > 1;
            }
            return g;
        };
        bool mn = tc_ok && bfd && lin_tm != nullptr;
        for (int d = 0; d < D && mn; ++d) {
            mn = tc_gemm_supported(mn_gemm(d, 0)) && (T < 2 || tc_gemm_supported(mn_gemm(d, 1))) &&
                 (!h0_v || tc_gemm_supported(mn_gemm(d, 2)));
        }
        if (mn) {
            for (int d = 0; d < D; ++d) {
                for (int which = 0; which < 3; ++which) {
                    const TcGemmArgs g = mn_gemm(d, which);
                    if ((which == 1 && T < 2) || (which == 2 && !h0_v)) continue;
                    int nl = 1;
                    LSTM_CUDA(timed(K_DW_TC, stream, [&] { return launch_tc_gemm(g, stream, &nl); }, &nl));
                }
                if (T < 2 && !h0_v) LSTM_CUDA(cudaMemsetAsync(dw_hh[k * D + d], 0, (size_t)G * H * 4, stream));
                TransposeArgs tww{};
                tww.M = G; tww.C = in; tww.mode = 0;
                tww.src = w_ih[k * D + d]; tww.lds = in; tww.src_bf16 = 1;
                tww.dst = wcatT + (size_t)d * G * wes; tww.ldd = (long long)D * G; tww.dst_bf16 = 1;
                LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] { return launch_transpose(tww, stream); }));
            }
            int nl = 1;
            LSTM_CUDA(timed(K_DX_TC, stream, [&] { return launch_tc_gemm(tx, stream, &nl); }, &nl));
        } else if (tc_ok) {
            TransposeArgs ta{};
            ta.M = (int)BTl; ta.C = D * G; ta.mode = 0; ta.src = dG; ta.lds = ldg; ta.src_bf16 = bfd;
            ta.dst = dGT; ta.ldd = BTl; ta.dst_bf16 = wbf;
            LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] { return launch_transpose(ta, stream); }));
            for (int d = 0; d < D; ++d) {
                char* bo = bop + (size_t)d * (in + H) * BTl * wes;
                TransposeArgs ti{};
                ti.M = (int)BTl; ti.C = in; ti.mode = 0;
                ti.src = lin_v; ti.lds = in; ti.src_bf16 = bfd;
                if (k == 0) {
                    ti.bt_remap = desc->batch_first; ti.T = T; ti.B = B;
                }
                ti.dst = bo; ti.ldd = BTl; ti.dst_bf16 = wbf;
                LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] { return launch_transpose(ti, stream); }));
                TransposeArgs th{};
                th.M = (int)BTl; th.C = H; th.mode = 1;
                th.src = static_cast<const char*>(hs_v) + (size_t)d * H * ses;
                th.lds = ldh; th.T = T; th.B = B; th.dir = d; th.src_bf16 = bfd;
                if (bfd)
                    th.h0 = h0 ? static_cast<const char*>(h0) + ((size_t)k * D + d) * B * H * 2 : nullptr;
                else
                    th.h0 = h0f ? h0f + ((size_t)k * D + d) * B * H : nullptr;
                th.dst = bo + (size_t)in * BTl * wes; th.ldd = BTl; th.dst_bf16 = wbf;
                LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] { return launch_transpose(th, stream); }));
                TcGemmArgs twd = tw;
                twd.A = dGT + (size_t)d * G * BTl * wes;
                twd.B = bo;
                twd.C = dw_ih[k * D + d];
                twd.C1 = dw_hh[k * D + d];
                if (overlap_dw && k > 0) {
                    deferred_dw.push_back(twd);   // launched behind layer k-1's recurrence
                } else {
                    int nl = 1;
                    LSTM_CUDA(timed(K_DW_TC, stream, [&] { return launch_tc_gemm(twd, stream, &nl); }, &nl));
                }
                TransposeArgs tww{};
                tww.M = G; tww.C = in; tww.mode = 0;
                tww.src = bfd ? w_ih[k * D + d] : static_cast<const void*>(wihf[k * D + d]);
                tww.lds = in; tww.src_bf16 = bfd;
                tww.dst = wcatT + (size_t)d * G * wes; tww.ldd = (long long)D * G; tww.dst_bf16 = wbf;
                LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] { return launch_transpose(tww, stream); }));
            }
            if (wbf && !bfd)
                LSTM_CUDA(timed(K_TRANSPOSE, stream, [&] {
                    return launch_convert(dG, DType::F32, dGT, DType::BF16, BTl * ldg, stream);
                }));
            {
                int nl = 1;
                LSTM_CUDA(timed(K_DX_TC, stream, [&] { return launch_tc_gemm(tx, stream, &nl); }, &nl));
            }
        } else {
            for (int d = 0; d < D; ++d) {
                // dW_ih = sum_t dG_t^T x_t
                GemmArgs g{};
                g.M = G; g.N = in; g.K = B * T;
                g.A = dG + (size_t)d * G; g.ta = DType::F32; g.sAm = 1; g.sAk = ldg;
                g.B = layer_in; g.tb = DType::F32; g.sBk = in; g.sBn = 1;
                g.C = dw_ih[k * D + d]; g.tc = DType::F32; g.ldc = in;
                LSTM_CUDA(timed(K_DW_SIMT, stream, [&] { return launch_gemm(g, stream); }));
                // dW_hh = sum_t dG_t^T h_{t-1} (h_{-1} = h0)
                GemmArgs gh{};
                gh.M = G; gh.N = H; gh.K = B * (T - 1);
                gh.ta = DType::F32; gh.sAm = 1; gh.sAk = ldg;
                gh.tb = DType::F32; gh.sBk = ldh; gh.sBn = 1;
                gh.C = dw_hh[k * D + d]; gh.tc = DType::F32; gh.ldc = H;
                if (d == 0) {
                    gh.A = dG + (size_t)B * ldg + (size_t)d * G;     // rows t >= 1
                    gh.B = hs + (size_t)d * H;                        // h at t-1
                } else {
                    gh.A = dG + (size_t)d * G;                        // rows t <= T-2
                    gh.B = hs + (size_t)B * ldh + (size_t)d * H;      // h at t+1
                }
                if (T > 1) {
                    LSTM_CUDA(timed(K_DW_SIMT, stream, [&] { return launch_gemm(gh, stream); }));
                } else {
                    LSTM_CUDA(cudaMemsetAsync(dw_hh[k * D + d], 0, (size_t)G * H * 4, stream));
                }
                if (h0f) {
                    GemmArgs g0 = gh;
                    g0.K = B;
                    g0.A = dG + (d == 0 ? 0 : (size_t)(T - 1) * B * ldg) + (size_t)d * G;
                    g0.B = h0f + ((size_t)k * D + d) * B * H;
                    g0.sBk = H;
                    g0.accumulate = 1;
                    LSTM_CUDA(timed(K_DW_SIMT, stream, [&] { return launch_gemm(g0, stream); }));
                }
            }
            // gradient w.r.t. the layer input: sum_d dG_d W_ih_d
            for (int d = 0; d < D; ++d) {
                GemmArgs g{};
                g.M = B * T; g.N = in; g.K = G;
                g.A = dG + (size_t)d * G; g.ta = DType::F32; g.sAm = ldg; g.sAk = 1;
                g.B = wihf[k * D + d]; g.tb = DType::F32; g.sBk = in; g.sBn = 1;
                g.C = din; g.tc = DType::F32; g.ldc = in;
                g.accumulate = d > 0;
                if (k == 0 && desc->batch_first) { g.remap_T = -T; g.remap_B = B; }
                LSTM_CUDA(timed(K_DX_SIMT, stream, [&] { return launch_gemm(g, stream); }));
            }
        }
        if (k > 0 && dropped) {   // through the dropout mask to layer k - 1's output
            const DropoutArgs da = dropout_args(desc, k - 1, din, din, DType::F32, (long long)BTl * in);
            LSTM_CUDA(timed(K_DROPOUT, stream, [&] { return launch_dropout(da, stream); }));
        }
        if (k > 0) {
            dy = din;
            dy_st = (long long)B * in;
            dy_sb = in;
            cur ^= 1;
        }
    }
    if (bf) {
        LSTM_CUDA(launch_convert(dxf, DType::F32, dx, DType::BF16, (long long)(BTs * l.I), stream));
        LSTM_CUDA(launch_convert(dh0f, DType::F32, dh0, DType::BF16, (long long)(L * state), stream));
    }
    (void)status;
    return LSTM_OK;
}

}  // extern "C"
