// liblstm.cu -- C ABI of liblstm (declared in include/liblstm.h): argument
// checks, workspace layout and the stream-ordered kernel sequence of the LSTM
// forward pass and its backpropagation through time ("SingleLayerLstmGrad").
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <algorithm>
#include <climits>
#include <cmath>
#include <cstdlib>
#include <mutex>
#include <vector>

#include "../../include/liblstm.h"
#include "../../include/liblstm_testing.h"
#include "common.cuh"
#include "simt.cuh"
#include "tc_host.cuh"
#include "tc_recur.cuh"
#include "tc_recur2.cuh"
#include "tc_recur3.cuh"
#include "tc_recur4.cuh"
#include "persist.cuh"

using namespace lstm;

namespace {

// ---------------------------------------------------------------- profiling
// Optional per-phase event pairs (lstm_profile_begin / lstm_profile_end).
namespace prof {
bool g_on = false;
struct Rec {
    int phase;
    cudaEvent_t a, b;
    long long launches;
};
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
    if (!g_pool.empty()) {
        cudaEvent_t e = g_pool.back();
        g_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// RAII scope: records an event before and after the phase's launches.
struct Phase {
    int phase;
    cudaStream_t s;
    cudaEvent_t a = nullptr;
    long long l0;
    Phase(int p, cudaStream_t st) : phase(p), s(st), l0(launch_counter().load()) {
        if (g_on && (a = take_event()) != nullptr) cudaEventRecord(a, s);
    }
    ~Phase() {
        if (!g_on || !a) return;
        cudaEvent_t b = take_event();
        if (!b) return;
        cudaEventRecord(b, s);
        g_recs.push_back({phase, a, b, launch_counter().load() - l0});
    }
};
}  // namespace prof

// ----------------------------------------------------- environment switches
// The library reads exactly these variables, at every call (no caching); the
// list, with defaults, is in include/liblstm_testing.h:
//   LSTM_FORCE_SIMT=1      CUDA-core kernels only
//   LSTM_FWD_FUSED_X=0     no fused forward kernel (the Gx plans)
//   LSTM_BWD_TMEM_W=0      no backward kernel with the weights in tensor memory
//   LSTM_BWD_STREAMS=1     that backward with one batch stream per group
//   LSTM_BWD_CHUNKS=n      reverse-time chunks of the overlapped backward
//   LSTM_PERSIST=0         no persistent CUDA-core recurrences (one launch per step)
//   LSTM_PERSIST_KS=n      their K split over clusters of n CTAs only (1, 2, 4, 8)
//   LSTM_STACK_WAVE=0      stacked layers one after another (no layer wavefront)
//   LSTM_STACK_CHUNKS=n    chunks per layer of the layer wavefront
//   LSTM_LAUNCH_NONCOOP=1  cluster launches without the cooperative attribute
//                          (also taken when a profiler or sanitizer is attached:
//                          NV_COMPUTE_PROFILER_PERFWORKS_DIR or
//                          CUDA_INJECTION64_PATH set)
bool env_is(const char *name, char value) {
    const char *e = getenv(name);
    return e && e[0] == value && e[1] == '\0';
}
bool force_simt() { return env_is("LSTM_FORCE_SIMT", '1'); }
// Persistent grids are launched without the cooperative attribute (after an
// occupancy check) when LSTM_LAUNCH_NONCOOP=1 or a profiler or sanitizer is
// attached: Nsight Compute sets NV_COMPUTE_PROFILER_PERFWORKS_DIR in the
// process it profiles, tools that inject through CUDA_INJECTION64_PATH set that.
bool profiler_attached() {
    const char *inj = getenv("CUDA_INJECTION64_PATH");
    const char *ncu = getenv("NV_COMPUTE_PROFILER_PERFWORKS_DIR");
    return env_is("LSTM_LAUNCH_NONCOOP", '1') || (inj && inj[0]) || (ncu && ncu[0]);
}

// ------------------------------------------------------------ validation
bool dims_ok(const lstm_dims *d) {
    if (!d) return false;
    if (d->T < 0 || d->B < 0 || d->I < 0 || d->H < 0) return false;
    if (d->dtype != LSTM_F32 && d->dtype != LSTM_BF16 && d->dtype != LSTM_F16) return false;
    const long long TB = (long long)d->T * d->B;
    const long long G4 = 4LL * d->H;
    const long long K = (long long)d->H + d->I;
    // every row / column index used by the kernels fits in an int
    if (TB > INT_MAX || G4 > INT_MAX || K > INT_MAX) return false;
    return true;
}

// Column extents beyond the 65535 x 64 columns one grid dimension covers.
bool dims_supported(const lstm_dims *d) {
    const long long maxcols = 65535LL * 64;
    return 4LL * d->H <= maxcols && (long long)d->H + d->I <= maxcols;
}

size_t esize(const lstm_dims *d) { return d->dtype == LSTM_F32 ? 4 : 2; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// A pointer argument: must be non-NULL when `needed`, and 16-byte aligned.
bool ptr_ok(const void *p, bool needed) {
    if (!p) return !needed;
    return aligned16(p);
}

struct FwdLayout {
    size_t gx, total;
};
FwdLayout fwd_layout(const lstm_dims *d) {
    FwdLayout L;
    const size_t TB = (size_t)d->T * d->B, G4 = 4 * (size_t)d->H;
    L.gx = kCtrlBytes;
    L.total = align_up(L.gx + TB * G4 * sizeof(float), 256);
    return L;
}

// db partial sums: at most kDbMaxChunks row chunks of >= 32 rows each (enough
// CTAs to cover the SMs at small T * B; one thread sums one column of a chunk).
constexpr long long kDbMaxChunks = 256;

// K splits of the CUDA-core dW GEMM (K = T*B rows): enough 64 x 64 output tiles
// times splits for about two CTAs per SM of a 148-SM part (a fixed target, so
// that the workspace size does not depend on the device), at most 8 splits of
// at least 256 rows each; 1 when the tiles alone fill the part.
constexpr long long kDwSplitTarget = 296;
int dw_splits(const lstm_dims *d) {
    const long long tiles = (4LL * d->H + 63) / 64 * ((long long)(d->H + d->I) + 63) / 64;
    const long long rows = (long long)d->T * d->B;
    if (tiles <= 0) return 1;
    long long S = std::min<long long>(8, (kDwSplitTarget + tiles - 1) / tiles);
    S = std::min<long long>(S, rows / 256);
    return (int)std::max<long long>(1, S);
}

struct BwdLayout {
    size_t dG, dc, dhp, dbpart, dwsplit, wt, dbgroup, total;
    int db_chunks, db_rows_per_chunk, dw_splits;
};
constexpr int kMaxGroups = 48;
BwdLayout bwd_layout(const lstm_dims *d) {
    BwdLayout L;
    const size_t TB = (size_t)d->T * d->B, G4 = 4 * (size_t)d->H;
    const size_t BH = (size_t)d->B * d->H;
    long long rows = 32;
    if ((long long)TB > rows * kDbMaxChunks) rows = ((long long)TB + kDbMaxChunks - 1) / kDbMaxChunks;
    L.db_rows_per_chunk = (int)rows;
    L.db_chunks = (int)(((long long)TB + rows - 1) / rows);
    L.dG = kCtrlBytes;
    L.dc = align_up(L.dG + TB * G4 * esize(d), 256);
    // delta h that padding passes to h_{t-1} (variable-length calls), ping-pong
    L.dhp = align_up(L.dc + 2 * BH * sizeof(float), 256);
    L.dbpart = align_up(L.dhp + 2 * BH * sizeof(float), 256);
    // partial products of the split-K CUDA-core dW GEMM
    L.dw_splits = dw_splits(d);
    L.dwsplit = align_up(L.dbpart + (size_t)L.db_chunks * G4 * sizeof(float), 256);
    const size_t dwpart = L.dw_splits > 1
                              ? (size_t)L.dw_splits * G4 * ((size_t)d->H + d->I) * sizeof(float)
                              : 0;
    L.wt = align_up(L.dwsplit + dwpart, 256);
    L.dbgroup = L.wt;
    L.total = L.wt;
    if (d->dtype != LSTM_F32) {
        // W_h^T [H][4H] and per-batch-group db partials of the persistent kernel
        L.dbgroup = align_up(L.wt + (size_t)d->H * G4 * 2, 256);
        L.total = align_up(L.dbgroup + (size_t)kMaxGroups * G4 * sizeof(float), 256);
    }
    return L;
}

// The tcgen05 GEMM core serves 16-bit (bf16 or fp16) problems whose rows are
// whole 16-byte groups (TMA strides and the W_x base offset are then 16-byte
// aligned).
bool tc_gemm_ok(const lstm_dims *d) {
    return !force_simt() && d->dtype != LSTM_F32 && d->H >= 8 && d->I >= 8 && d->H % 8 == 0 &&
           d->I % 8 == 0 && tcg::encode_fn() != nullptr;
}

int ws_ok(void *ws, size_t ws_bytes, size_t need) {
    if (!ws || ws_bytes < need || ((uintptr_t)ws & 255u) != 0) return LSTM_ERR_WORKSPACE;
    return LSTM_OK;
}

#define LSTM_TRY(expr)                                    \
    do {                                                  \
        cudaError_t e_ = (expr);                          \
        if (e_ != cudaSuccess) return LSTM_ERR_CUDA;      \
    } while (0)

cudaError_t reset_barriers(void *ws, cudaStream_t s) {
    // the whole control block: status word, failing site and barrier counters
    // (a workspace fresh from an allocator holds anything)
    return cudaMemsetAsync(ws, 0, kCtrlBytes, s);
}

template <class T>
cudaError_t launch_copy_or_zero(const T *in, T *out, long long n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    simt::copy_or_zero<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(in, out, n);
    note_launch();
    return cudaGetLastError();
}

template <class T>
cudaError_t launch_to_float(const T *in, float *out, long long n, cudaStream_t s) {
    if (n <= 0) return cudaSuccess;
    simt::to_float_copy<T><<<(unsigned)((n + 255) / 256), 256, 0, s>>>(in, out, n);
    note_launch();
    return cudaGetLastError();
}

// ------------------------------------------- tensor-core GEMM problems
typedef __nv_bfloat16 bf16;

// The 16-bit type the tensor-core paths of fwd_simt<T> / bwd_simt<T> use: T
// itself for bf16 and fp16 (float never reaches them).
template <class T> struct Tc16 { typedef T type; };
template <> struct Tc16<float> { typedef bf16 type; };

// a1 on tcgen05: Gx[TB][4H] = X[TB][I] W_x^T + b, both operands K-major.
template <class E>
cudaError_t tc_input_projection(const lstm_dims *d, const E *x, const E *W, const E *b,
                                float *Gx, Ctrl *ctrl, cudaStream_t s) {
    const long long TB = (long long)d->T * d->B, H = d->H, I = d->I;
    tcg::Builder bld(ctrl, Elem<E>::kFmt);
    const int mx = bld.add_map({x, TB, I, I}, 0, tcg::BM);
    const int mw = bld.add_map({W + H, 4 * H, I, H + I}, 0, tcg::BN);
    tcg::Problem &q = bld.add_problem((int)TB, (int)(4 * H), 0, 0, Gx, 4 * H, 0, b);
    tcg::Builder::add_seg(q, mx, 0, mw, 0, I);
    if (!bld.ok) return cudaErrorInvalidValue;
    return tcg::launch(bld, s);
}

// a4 + a6 on tcgen05 in one persistent launch:
//   dW[:, 0:H]  = dG[B:]^T y[:-B] + dG[:B]^T h0   (h_prev = [h0; y[0:T-1]])
//   dW[:, H:]   = dG^T X
//   dx          = dG W_x
// dG^T and the z-rows are MN-major operands read straight from their
// row-major storage; the time shift of h_prev is a TMA row offset.
// a4 + a6 over the rows of time steps [t_lo, t_hi):
//   dW (+)= dG[rows]^T [h_prev | x][rows],   dx[rows] = dG[rows] W_x.
// The operand maps end at the range's last row, so a partial 64-row K block
// reads zeros rather than rows of the next range.  At most max_ctas CTAs
// (0: one per SM).  parts: DW_PART and / or DX_PART.
constexpr int DW_PART = 1, DX_PART = 2;
template <class E>
cudaError_t tc_dw_dx(const lstm_dims *d, const E *dG, const E *x, const E *W, const E *h0,
                     const E *y, float *dW, float *dx, Ctrl *ctrl, cudaStream_t s, int t_lo,
                     int t_hi, bool accumulate, int max_ctas, bool reverse = false,
                     int parts = DW_PART | DX_PART) {
    const long long B = d->B, H = d->H, I = d->I, G4 = 4 * H;
    const long long r0 = (long long)t_lo * B, r1 = (long long)t_hi * B;
    tcg::Builder bld(ctrl, Elem<E>::kFmt);
    if (parts & DX_PART) {  // dx rows r0 .. r1-1 first in the tile queue
        const int m_dg_k = bld.add_map({dG, r1, G4, G4}, 0, tcg::BM);
        const int m_wx_mn = bld.add_map({W + H, G4, I, H + I}, 1, 0);
        tcg::Problem &p2 = bld.add_problem((int)(r1 - r0), (int)I, 0, 1, dx + r0 * I, I, 0,
                                           nullptr);
        p2.a_mn0 = (int)r0;
        tcg::Builder::add_seg(p2, m_dg_k, 0, m_wx_mn, 0, G4);
    }
    if (!(parts & DW_PART)) {
        if (!bld.ok) return cudaErrorInvalidValue;
        return tcg::launch(bld, s, max_ctas);
    }
    const int m_dg_mn = bld.add_map({dG, r1, G4, G4}, 1, 0);
    const int m_x_mn = bld.add_map({x, r1, I, I}, 1, 0);
    tcg::Problem &p0 = bld.add_problem((int)G4, (int)H, 1, 1, dW, H + I, 0, nullptr);
    p0.accumulate = accumulate;
    if (!reverse) {
        // h_prev of row r is y row r - B (r >= B) or h0 row r (r < B, only when t_lo == 0)
        const long long ry0 = std::max(r0, B);
        const int m_y_mn = (r1 > ry0) ? bld.add_map({y, r1 - B, H, H}, 1, 0) : -1;
        const int m_h0_mn = (h0 && r0 < B) ? bld.add_map({h0, B, H, H}, 1, 0) : -1;
        // dW, h-part (no K segment, i.e. zero, when the range is t = 0 alone and h0 is absent)
        if (m_y_mn >= 0)
            tcg::Builder::add_seg(p0, m_dg_mn, (int)ry0, m_y_mn, (int)(ry0 - B), r1 - ry0);
        if (m_h0_mn >= 0) tcg::Builder::add_seg(p0, m_dg_mn, 0, m_h0_mn, 0, B);
    } else {
        // reverse direction: h_prev of row r is y row r + B (r < last0 = (T-1) B) or
        // h0 row r - last0 (the last time, only when t_hi == T)
        const long long last0 = (long long)(d->T - 1) * B;
        const long long ry1 = std::min(r1, last0);
        const int m_y_mn = (ry1 > r0) ? bld.add_map({y, ry1 + B, H, H}, 1, 0) : -1;
        const int m_h0_mn = (h0 && r1 > last0) ? bld.add_map({h0, B, H, H}, 1, 0) : -1;
        if (m_y_mn >= 0)
            tcg::Builder::add_seg(p0, m_dg_mn, (int)r0, m_y_mn, (int)(r0 + B), ry1 - r0);
        if (m_h0_mn >= 0) tcg::Builder::add_seg(p0, m_dg_mn, (int)last0, m_h0_mn, 0, B);
    }
    // dW, x-part
    tcg::Problem &p1 = bld.add_problem((int)G4, (int)I, 1, 1, dW, H + I, (int)H, nullptr);
    p1.accumulate = accumulate;
    tcg::Builder::add_seg(p1, m_dg_mn, (int)r0, m_x_mn, (int)r0, r1 - r0);
    if (!bld.ok) return cudaErrorInvalidValue;
    return tcg::launch(bld, s, max_ctas);
}

// Streams of a chunked backward call, per device: the recurrence on a
// high-priority stream (its clusters are placed before pending GEMM CTAs),
// the dW / dx GEMMs on a low-priority one, joined back into the caller's
// stream with events.  Created on first use and kept for the process.
constexpr int kMaxChunks = 16;
struct AuxStreams {
    cudaStream_t rec = nullptr, gemm = nullptr;
    cudaEvent_t ev[kMaxChunks + 3] = {};
    bool ready = false, tried = false;
    std::mutex mu;  // one chunked call enqueues at a time (the events are shared)
};

AuxStreams *aux_streams() {
    static std::mutex mu;
    static AuxStreams per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    AuxStreams &a = per_dev[dev];
    if (!a.tried) {
        a.tried = true;
        int lo = 0, hi = 0;
        bool ok = cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&a.rec, cudaStreamNonBlocking, hi) == cudaSuccess &&
                  cudaStreamCreateWithPriority(&a.gemm, cudaStreamNonBlocking, lo) == cudaSuccess;
        for (int i = 0; ok && i < kMaxChunks + 3; ++i)
            ok = cudaEventCreateWithFlags(&a.ev[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) cudaGetLastError();
        a.ready = ok;
    }
    return a.ready ? &a : nullptr;
}

// Streams and events of the stacked forward's layer wavefront: one stream per
// layer (layers past kMaxWave share them in turn), an event per (layer stream,
// chunk), and the fork / join events.
constexpr int kMaxWave = 8, kMaxWaveChunks = 8;
struct WaveStreams {
    cudaStream_t st[kMaxWave] = {};
    cudaEvent_t ev[kMaxWave][kMaxWaveChunks] = {};
    cudaEvent_t fork = nullptr, join[kMaxWave] = {};
    bool ready = false, tried = false;
    std::mutex mu;  // one wavefront call enqueues at a time (the events are shared)
};

WaveStreams *wave_streams() {
    static std::mutex mu;
    static WaveStreams per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    WaveStreams &w = per_dev[dev];
    if (!w.tried) {
        w.tried = true;
        bool ok = cudaEventCreateWithFlags(&w.fork, cudaEventDisableTiming) == cudaSuccess;
        for (int l = 0; ok && l < kMaxWave; ++l) {
            ok = cudaStreamCreateWithFlags(&w.st[l], cudaStreamNonBlocking) == cudaSuccess &&
                 cudaEventCreateWithFlags(&w.join[l], cudaEventDisableTiming) == cudaSuccess;
            for (int c = 0; ok && c < kMaxWaveChunks; ++c)
                ok = cudaEventCreateWithFlags(&w.ev[l][c], cudaEventDisableTiming) == cudaSuccess;
        }
        if (!ok) cudaGetLastError();
        w.ready = ok;
    }
    return w.ready ? &w : nullptr;
}

// Streams and events of the stacked backward's layer wavefront, per layer:
// the recurrence (highest priority), the dx GEMM that feeds the layer below
// (highest priority), and the dW GEMM (lowest), with an event per (layer,
// chunk) for a finished recurrence chunk and for the next lower layer's dy
// rows of that chunk.
struct WaveBwdStreams {
    cudaStream_t rec[kMaxWave] = {}, dxs[kMaxWave] = {}, gemm[kMaxWave] = {};
    cudaEvent_t ev_rec[kMaxWave][kMaxChunks] = {}, ev_dy[kMaxWave][kMaxChunks] = {};
    cudaEvent_t fork = nullptr, join[3 * kMaxWave] = {};
    bool ready = false, tried = false;
    std::mutex mu;
};

WaveBwdStreams *wave_bwd_streams() {
    static std::mutex mu;
    static WaveBwdStreams per_dev[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> g(mu);
    WaveBwdStreams &w = per_dev[dev];
    if (!w.tried) {
        w.tried = true;
        int lo = 0, hi = 0;
        bool ok = cudaDeviceGetStreamPriorityRange(&lo, &hi) == cudaSuccess &&
                  cudaEventCreateWithFlags(&w.fork, cudaEventDisableTiming) == cudaSuccess;
        for (int l = 0; ok && l < kMaxWave; ++l) {
            ok = cudaStreamCreateWithPriority(&w.rec[l], cudaStreamNonBlocking, hi) == cudaSuccess &&
                 cudaStreamCreateWithPriority(&w.dxs[l], cudaStreamNonBlocking, hi) == cudaSuccess &&
                 cudaStreamCreateWithPriority(&w.gemm[l], cudaStreamNonBlocking, lo) == cudaSuccess;
            for (int c = 0; ok && c < kMaxChunks; ++c)
                ok = cudaEventCreateWithFlags(&w.ev_rec[l][c], cudaEventDisableTiming) == cudaSuccess &&
                     cudaEventCreateWithFlags(&w.ev_dy[l][c], cudaEventDisableTiming) == cudaSuccess;
        }
        for (int i = 0; ok && i < 3 * kMaxWave; ++i)
            ok = cudaEventCreateWithFlags(&w.join[i], cudaEventDisableTiming) == cudaSuccess;
        if (!ok) cudaGetLastError();
        w.ready = ok;
    }
    return w.ready ? &w : nullptr;
}

// Number of reverse-time chunks of a backward call whose dW / dx GEMMs run
// beside the recurrence (1: no overlap): at least 16 steps per chunk, at most
// 6 chunks (the last chunk's GEMM is the part that cannot overlap; each chunk
// costs one more launch of the recurrence, with its weights loaded again).
// LSTM_BWD_CHUNKS overrides.
int bwd_chunks(const lstm_dims *d) {
    const char *e = getenv("LSTM_BWD_CHUNKS");
    int n = e ? atoi(e) : (d->T >= 32 ? std::min(6, d->T / 16) : 1);
    return std::max(1, std::min(std::min(n, kMaxChunks), d->T));
}

// First epilogue iteration of chunk c of nch over T steps (c = nch gives T).
// Chunk sizes shrink geometrically (ratio 0.8): the dW / dx GEMM of a chunk
// runs beside the next, smaller one, and the GEMM of the last chunk, which
// runs alone, is the smallest.  Every chunk keeps at least one step.
int chunk_bound(int T, int nch, int c) {
    constexpr double r = 0.8;
    if (c <= 0) return 0;
    if (c >= nch) return T;
    const double f = (1.0 - pow(r, c)) / (1.0 - pow(r, nch));
    int b = (int)(T * f + 0.5);
    b = std::max(b, c);               // at least one step per earlier chunk
    return std::min(b, T - (nch - c));  // and per later one
}

// ------------------------------------------- persistent recurrence (bf16)
// Test hooks (include/liblstm_testing.h): one CTA that never arrives, and the
// bound of every device-side wait.
int g_fault_skip_cta = -1;
// Which recurrent kernel the last lstm_fwd / lstm_bwd used (test hook):
// 0 per-step CUDA-core kernels, 1 persistent K-resident kernel, 2 cluster kernel.
int g_last_fwd_path = -1, g_last_bwd_path = -1;
int g_last_stack_chunks = -1;      // chunks per layer of the last stack forward's wavefront
int g_last_stack_bwd_chunks = -1;  // and of the last stack backward's
unsigned long long g_wait_ns = 2000000000ull;

struct RecPlan {
    int S, G, NB, kch, stages;
    size_t smem;
};

constexpr size_t kMaxSmem = 227 * 1024;

// Grid of the persistent forward recurrence: S = H/16 unit slices times G
// batch groups of NB rows (NB a power of two in 16..128), S*G <= SM count.
bool plan_fwd_recur(const lstm_dims *d, RecPlan &P) {
    // (the kernel reads W through a tensor map: rows of H + I elements must be
    // whole 16-byte groups)
    if (d->dtype != LSTM_BF16 || d->H % rec::UNITS != 0 || d->H > 1024 || d->B < 1 ||
        (d->H + d->I) % 8 != 0 || tcg::encode_fn() == nullptr)
        return false;
    if (force_simt()) return false;
    P.S = d->H / rec::UNITS;
    const int gmax = tcg::sm_count() / P.S;
    if (gmax < 1) return false;
    int G = std::min(gmax, (d->B + 15) / 16);
    int NB = 16;
    while (NB < (d->B + G - 1) / G) NB *= 2;
    if (NB > 128) return false;
    P.G = (d->B + NB - 1) / NB;
    if (P.G > gmax || P.G > 48) return false;
    P.NB = NB;
    P.kch = (d->H + 63) / 64;
    const size_t fixed = rec::FwdSmem(P.kch, 0, NB).total + 1024;
    const size_t per_stage = (size_t)NB * 128;
    if (fixed + 2 * per_stage > kMaxSmem) return false;
    P.stages = (int)std::min<size_t>(rec::MAX_STAGES, (kMaxSmem - fixed) / per_stage);
    P.smem = rec::FwdSmem(P.kch, P.stages, NB).total + 1024;
    return true;
}

template <int NB>
cudaError_t launch_fwd_recur(const rec::FwdParams &prm, int grid, size_t smem, cudaStream_t s) {
    static size_t attr_smem = 0;
    if (attr_smem < smem) {
        cudaError_t e = cudaFuncSetAttribute(rec::fwd_kernel<NB>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        attr_smem = smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(rec::NUM_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;  // all CTAs co-resident, or the launch fails
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, rec::fwd_kernel<NB>, prm);
    note_launch();
    return e;
}

// a2 as one persistent cooperative launch (see tc_recur.cuh).
int tc_fwd_recurrence(const lstm_dims *d, const RecPlan &P, const bf16 *W, const bf16 *h0,
                      const float *c0, const float *Gx, bf16 *y, bf16 *hT, float *cT, bf16 *gates,
                      float *cells, Ctrl *ctrl, cudaStream_t s) {
    const long long T = d->T, B = d->B, H = d->H, I = d->I;
    rec::FwdParams prm;
    memset(&prm, 0, sizeof(prm));
    bool ok = tcg::make_map(&prm.map_w, W, H + I, 4 * H, (H + I) * 2, 64, rec::UNITS) &&
              tcg::make_map(&prm.map_y, y, H, T * B, H * 2, 64, P.NB);
    if (h0) ok = ok && tcg::make_map(&prm.map_h0, h0, H, B, H * 2, 64, P.NB);
    else prm.map_h0 = prm.map_y;
    if (!ok) return LSTM_ERR_UNSUPPORTED;
    prm.Gx = Gx; prm.c0 = c0; prm.y = y; prm.gates = gates; prm.hT = hT;
    prm.cells = cells; prm.cT = cT; prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.S = P.S; prm.G = P.G;
    prm.kch = P.kch; prm.stages = P.stages; prm.has_h0 = h0 != nullptr;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const int grid = P.S * P.G;
    cudaError_t e;
    switch (P.NB) {
        case 16: e = launch_fwd_recur<16>(prm, grid, P.smem, s); break;
        case 32: e = launch_fwd_recur<32>(prm, grid, P.smem, s); break;
        case 64: e = launch_fwd_recur<64>(prm, grid, P.smem, s); break;
        default: e = launch_fwd_recur<128>(prm, grid, P.smem, s); break;
    }
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// Grid of the persistent backward recurrence: S = H/16 unit slices times G
// batch groups of NB <= 64 rows (the MMA's M is 64), S*G <= SM count.
bool plan_bwd_recur(const lstm_dims *d, RecPlan &P) {
    if (d->dtype != LSTM_BF16 || d->H % rec::UNITS != 0 || d->H > 1024 || d->B < 1 ||
        tcg::encode_fn() == nullptr)
        return false;
    if (force_simt()) return false;
    P.S = d->H / rec::UNITS;
    const int gmax = std::min(tcg::sm_count() / P.S, kMaxGroups);
    if (gmax < 1) return false;
    int G = std::min(gmax, (d->B + 15) / 16);
    int NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    if (NB > 64) {
        G = (d->B + 63) / 64;
        NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    }
    P.G = (d->B + NB - 1) / NB;
    if (P.G > gmax) return false;
    P.NB = NB;
    P.kch = 4 * d->H / 64;
    const size_t fixed = rec::BwdSmem(P.kch, 0).total + 1024;
    if (fixed + 2 * rec::BWD_STAGE_BYTES > kMaxSmem) return false;
    P.stages = (int)std::min<size_t>(rec::MAX_STAGES, (kMaxSmem - fixed) / rec::BWD_STAGE_BYTES);
    P.smem = rec::BwdSmem(P.kch, P.stages).total + 1024;
    return true;
}

// a3 (+ a5) as one persistent cooperative launch (see tc_recur.cuh); W_h^T is
// written to the workspace first, and db is the sum of the groups' partials.
int tc_bwd_recurrence(const lstm_dims *d, const RecPlan &P, const bf16 *dy, const bf16 *dhT,
                      const float *dcT, const bf16 *W, const float *c0, const bf16 *gates,
                      const float *cells, bf16 *dG, bf16 *WT, float *dbgroup, float *db,
                      float *dh0, float *dc0, Ctrl *ctrl, cudaStream_t s) {
    const long long T = d->T, B = d->B, H = d->H, I = d->I, G4 = 4 * H;
    {
        dim3 grid((unsigned)((H + 31) / 32), (unsigned)((G4 + 31) / 32));
        rec::transpose_wh<<<grid, dim3(32, 8), 0, s>>>(W, WT, (int)H, (int)I);
        note_launch();
        if (cudaGetLastError() != cudaSuccess) return LSTM_ERR_CUDA;
    }
    rec::BwdParams prm;
    memset(&prm, 0, sizeof(prm));
    if (!tcg::make_map(&prm.map_wt, WT, G4, H, G4 * 2, 64, rec::UNITS) ||
        !tcg::make_map(&prm.map_dg, dG, G4, T * B, G4 * 2, 64, P.NB))
        return LSTM_ERR_UNSUPPORTED;
    prm.dy = dy; prm.dhT = dhT; prm.gates = gates; prm.dcT = dcT; prm.cells = cells;
    prm.c0 = c0; prm.dG = dG; prm.dh0 = dh0; prm.dc0 = dc0; prm.db_part = dbgroup;
    prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.S = P.S; prm.G = P.G; prm.NB = P.NB;
    prm.kch4 = P.kch; prm.stages = P.stages;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    static size_t attr_smem = 0;
    if (attr_smem < P.smem) {
        if (cudaFuncSetAttribute(rec::bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)P.smem) != cudaSuccess)
            return LSTM_ERR_CUDA;
        attr_smem = P.smem;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(P.S * P.G);
    cfg.blockDim = dim3(rec::NUM_THREADS);
    cfg.dynamicSmemBytes = P.smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, rec::bwd_kernel, prm);
    note_launch();
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    if (e != cudaSuccess) return LSTM_ERR_CUDA;
    simt::colsum_final<<<(unsigned)((G4 + 255) / 256), 256, 0, s>>>(dbgroup, P.G, (int)G4, db);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// --------------------------------------- cluster recurrence kernels (bf16)
struct Rec2Plan {
    int KS, G, NB, kcc, R, stages;
    int kcx;  // fused forward: K chunks of x per CTA
    size_t smem;
    int split = 1;  // fused forward: batch streams per cluster (NB rows each)
    int family = 3; // backward with the weights in TMEM: 3, or 4 with two stream agents each
};

int max_active_clusters(const void *kern, int threads, size_t smem, int KS) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(KS);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = KS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

const void *fwd2_kernel_ptr(int NB, int KS) {
#define LSTM_F2(nb, ks) \
    if (NB == nb && KS == ks) return (const void *)rec2::fwd2_kernel<nb, ks>;
    LSTM_F2(16, 1) LSTM_F2(16, 2) LSTM_F2(16, 4)
    LSTM_F2(32, 1) LSTM_F2(32, 2) LSTM_F2(32, 4) LSTM_F2(32, 8)
    LSTM_F2(64, 2) LSTM_F2(64, 4) LSTM_F2(64, 8)
    LSTM_F2(128, 4) LSTM_F2(128, 8)
#undef LSTM_F2
    return nullptr;
}

// Forward: R = H/32 row slices x KS K-parts x G batch groups of NB rows;
// R * G clusters of KS must be co-resident.
bool plan_fwd2(const lstm_dims *d, Rec2Plan &P) {
    // (W through a tensor map: rows of H + I elements in whole 16-byte groups)
    if (d->dtype != LSTM_BF16 || d->H % rec2::F_UNITS != 0 || d->B < 1 ||
        (d->H + d->I) % 8 != 0 || tcg::encode_fn() == nullptr || force_simt())
        return false;
    const int nsm = tcg::sm_count();
    P.R = d->H / rec2::F_UNITS;
    for (int KS : {4, 2, 8, 1}) {
        if ((d->H / KS) % 64 != 0 || d->H % KS != 0) continue;
        const int kcc = d->H / KS / 64;
        if (kcc < 1 || kcc > rec2::MAX_KCC) continue;
        const int gsm = std::min(nsm / (P.R * KS), kMaxGroups);  // SM bound first
        if (gsm < 1) continue;
        const int G0 = std::min(gsm, (d->B + 15) / 16);
        int NB = 16;
        while (NB < (d->B + G0 - 1) / G0) NB *= 2;
        NB = std::max(NB, 4 * KS);
        if (NB > 128 || NB / KS > 32) continue;
        const int G = (d->B + NB - 1) / NB;
        const size_t smem = rec2::Fwd2Smem(kcc, NB, KS).total + 1024;
        if (smem > kMaxSmem) continue;
        const void *kern = fwd2_kernel_ptr(NB, KS);
        if (!kern) continue;
        const int maxc = max_active_clusters(kern, rec2::F_THREADS, smem, KS);
        if (G * P.R > maxc) continue;
        P.KS = KS; P.G = G; P.NB = NB; P.kcc = kcc; P.smem = smem;
        return true;
    }
    return false;
}

// Instantiations of the fused forward: (NB, KS) with one batch stream, and
// (NB, KS) per stream with two.
#define LSTM_F3_SPLIT1(X) X(16, 1) X(16, 2) X(16, 4) X(32, 1) X(32, 2) X(32, 4) X(32, 8) \
    X(64, 2) X(64, 4) X(64, 8) X(128, 4) X(128, 8)
#define LSTM_F3_SPLIT2(X) X(32, 2) X(32, 4) X(32, 8) X(64, 4) X(64, 8)

template <class E>
const void *fwd3_kernel_ptr(int NB, int KS, bool masked, int split) {
#define LSTM_F3(nb, ks)                                                                    \
    if (NB == nb && KS == ks)                                                              \
        return masked ? (const void *)rec3::fwd3_kernel<E, nb, ks, true, SPLIT_>           \
                      : (const void *)rec3::fwd3_kernel<E, nb, ks, false, SPLIT_>;
    if (split == 1) {
        constexpr int SPLIT_ = 1;
        LSTM_F3_SPLIT1(LSTM_F3)
    } else if (split == 2) {
        constexpr int SPLIT_ = 2;
        LSTM_F3_SPLIT2(LSTM_F3)
    }
#undef LSTM_F3
    return nullptr;
}

// Forward with the input projection fused: the grid of plan_fwd2, and the
// CTA's W_h and W_x K-slices must fit TMEM beside two accumulators.
// LSTM_FWD_FUSED_X=0 turns it off (comparison runs).
// share > 1: the plan takes at most 1/share of the SMs and of the clusters
// that can be co-resident (a layer of a stacked wavefront runs beside
// another layer's launch).
bool plan_fwd3(const lstm_dims *d, Rec2Plan &P, bool masked, int share = 1) {
    if (env_is("LSTM_FWD_FUSED_X", '0')) return false;
    if (d->dtype == LSTM_F32 || d->H % rec2::F_UNITS != 0 || d->B < 1 || d->I < 1 ||
        d->I % 8 != 0 || tcg::encode_fn() == nullptr || force_simt())
        return false;
    const int nsm = tcg::sm_count() / share;
    P.R = d->H / rec2::F_UNITS;
    for (int KS : {4, 2, 8, 1}) {
        if ((d->H / KS) % 64 != 0 || d->H % KS != 0) continue;
        const int kcc = d->H / KS / 64;
        const int kcx = (d->I + KS * 64 - 1) / (KS * 64);
        if (kcc < 1 || kcc > rec3::F3_MAXC || kcx > rec3::F3_MAXC) continue;
        const int gsm = std::min(nsm / (P.R * KS), kMaxGroups);  // SM bound first
        if (gsm < 1) continue;
        const int G0 = std::min(gsm, (d->B + 15) / 16);
        int NB = 16;
        while (NB < (d->B + G0 - 1) / G0) NB *= 2;
        NB = std::max(NB, 4 * KS);
        if (NB > 128 || NB / KS > 32) continue;
        const int G = (d->B + NB - 1) / NB;
        // two interleaved batch streams of NB / 2 rows per cluster where that
        // instantiation exists and fits, else one
        for (int split : {2, 1}) {
            if (split == 2 && (NB < 64 || G * 2 > kMaxGroups)) continue;
            const int NBv = NB / split;
            if (NBv / KS < 4) continue;
            if (rec3::fwd3_tmem_cols(NBv, kcc, kcx) > 512) continue;
            const size_t smem = rec3::Fwd3Smem(kcc, kcx, NBv, KS, split).total + 1024;
            if (smem > kMaxSmem) continue;
            const void *kern = d->dtype == LSTM_F16
                                   ? fwd3_kernel_ptr<__half>(NBv, KS, masked, split)
                                   : fwd3_kernel_ptr<bf16>(NBv, KS, masked, split);
            if (!kern) continue;
            const int maxc = max_active_clusters(kern, rec2::F_THREADS, smem, KS);
            if (G * P.R > maxc / share) continue;
            P.KS = KS; P.G = G; P.NB = NBv; P.kcc = kcc; P.kcx = kcx; P.smem = smem;
            P.split = split;
            P.family = 3;
            return true;
        }
    }
    return false;
}

// Backward: U = H/128 unit slices x 8 K-parts of 4H x G batch groups of NB rows;
// U * G clusters of 8 must be co-resident (cudaOccupancyMaxActiveClusters).
bool plan_bwd2(const lstm_dims *d, Rec2Plan &P) {
    if (d->dtype != LSTM_BF16 || d->H % rec2::B_UNITS != 0 || d->B < 1 ||
        tcg::encode_fn() == nullptr || force_simt())
        return false;
    P.KS = rec2::B_KS;
    P.R = d->H / rec2::B_UNITS;
    P.kcc = 4 * d->H / rec2::B_KS / 64;
    if (P.kcc < 1 || P.kcc > rec2::MAX_KCC) return false;
    const size_t fixed = rec2::Bwd2Smem(P.kcc, 0).total + 1024;
    if (fixed + 2 * rec2::B_ACHUNK > kMaxSmem) return false;
    // At least two stages: the ring also stages the first exchange round
    // (B_ROUND0 partners x 8 KB = 32 KB) between an iteration's last MMA and the
    // next iteration's loads.
    const int stages = (int)std::min<size_t>(std::max(2, std::min(P.kcc, rec2::MAX_KCC)),
                                             (kMaxSmem - fixed) / rec2::B_ACHUNK);
    if (stages < 2 || (size_t)stages * rec2::B_ACHUNK < rec2::B_STAGE_BYTES) return false;
    P.NB = stages;  // (ring stages; NB is reassigned to the batch rows below)
    P.smem = rec2::Bwd2Smem(P.kcc, stages).total + 1024;
    const int maxc = max_active_clusters((const void *)rec2::bwd2_kernel, rec2::B_THREADS, P.smem,
                                         P.KS);
    const int gmax = std::min(maxc / P.R, kMaxGroups);
    if (gmax < 1) return false;
    int G = std::min(gmax, (d->B + 15) / 16);
    int NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    if (NB > rec2::B_MROWS) {
        G = (d->B + rec2::B_MROWS - 1) / rec2::B_MROWS;
        NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    }
    P.G = (d->B + NB - 1) / NB;
    if (P.G > gmax) return false;
    P.stages = stages;
    P.NB = NB;
    return true;
}

// Backward with W_h^T in TMEM: same grid as plan_bwd2; the K slice (H/2) must
// fit TMEM beside the accumulator (H <= 1536) and the ring must stage one
// exchange round (at least 4 stages, H >= 512).  LSTM_BWD_TMEM_W=0 turns it
// off (comparison runs).
bool plan_bwd3(const lstm_dims *d, Rec2Plan &P, int share = 1) {
    if (env_is("LSTM_BWD_TMEM_W", '0')) return false;
    if (d->dtype == LSTM_F32 || d->H % rec3::UNITS != 0 || d->B < 1 ||
        tcg::encode_fn() == nullptr || force_simt())
        return false;
    P.KS = rec3::KS;
    P.R = d->H / rec3::UNITS;
    P.kcc = 4 * d->H / rec3::KS / 64;
    if (rec3::W_COL + (uint32_t)(P.kcc * 32) > rec3::TMEM_COLS) return false;
    int stages = std::min(P.kcc, rec3::MAX_STAGES);
    while (stages >= rec3::MIN_STAGES && (size_t)rec3::Bwd3Smem(stages).total + 1024 > kMaxSmem) --stages;
    if (stages < rec3::MIN_STAGES) return false;
    P.smem = rec3::Bwd3Smem(stages).total + 1024;
    const void *kern = d->dtype == LSTM_F16 ? (const void *)rec3::bwd3_kernel<__half, false, false>
                                            : (const void *)rec3::bwd3_kernel<bf16, false, false>;
    const int maxc = max_active_clusters(kern, rec3::THREADS, P.smem, P.KS);
    const int gmax = std::min(std::min(maxc / share / P.R, kMaxGroups),
                              tcg::sm_count() / share / (P.R * P.KS));
    if (gmax < 1) return false;
    int G = std::min(gmax, (d->B + 15) / 16);
    int NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    if (NB > rec3::NMAX) {
        G = (d->B + rec3::NMAX - 1) / rec3::NMAX;
        NB = ((d->B + G - 1) / G + 15) / 16 * 16;
    }
    P.G = (d->B + NB - 1) / NB;
    if (P.G > gmax) return false;
    P.stages = stages;
    P.NB = NB;
    P.family = 3;
    return true;
}

// Backward with two decoupled batch streams per group (rec4): the grid of
// plan_bwd3 with groups of a multiple of 32 rows (two streams of a multiple of
// 16), 384 threads, and each stream's ring staging its send blocks.
bool plan_bwd4(const lstm_dims *d, Rec2Plan &P, int share = 1) {
    if (env_is("LSTM_BWD_TMEM_W", '0') || env_is("LSTM_BWD_STREAMS", '1')) return false;
    if (d->dtype == LSTM_F32 || d->H % rec4::UNITS != 0 || d->B < 1 ||
        tcg::encode_fn() == nullptr || force_simt())
        return false;
    P.KS = rec4::KS;
    P.R = d->H / rec4::UNITS;
    P.kcc = 4 * d->H / rec4::KS / 64;
    if (rec4::W_COL + (uint32_t)(P.kcc * 32) > rec4::TMEM_COLS) return false;
    int stages = std::min(P.kcc, rec4::MAX_STAGES);
    while (stages >= rec4::MIN_STAGES && (size_t)rec4::Bwd4Smem(stages).total + 1024 > kMaxSmem)
        --stages;
    if (stages < rec4::MIN_STAGES) return false;
    P.smem = rec4::Bwd4Smem(stages).total + 1024;
    const void *kern = d->dtype == LSTM_F16 ? (const void *)rec4::bwd4_kernel<__half, false, false>
                                            : (const void *)rec4::bwd4_kernel<bf16, false, false>;
    const int maxc = max_active_clusters(kern, rec4::THREADS, P.smem, P.KS);
    const int gmax = std::min(std::min(maxc / share / P.R, kMaxGroups / rec4::NSTREAM),
                              tcg::sm_count() / share / (P.R * P.KS));
    if (gmax < 1) return false;
    const int rows_max = rec4::NSTREAM * rec4::NBS_MAX;
    int G = std::min(gmax, (d->B + 31) / 32);
    int NB = ((d->B + G - 1) / G + 31) / 32 * 32;
    if (NB > rows_max) {
        G = (d->B + rows_max - 1) / rows_max;
        NB = ((d->B + G - 1) / G + 31) / 32 * 32;
    }
    P.G = (d->B + NB - 1) / NB;
    if (P.G > gmax) return false;
    // both streams of every group hold rows (else the one-stream kernel serves)
    if (d->B <= (NB / 2) * (2 * P.G - 1)) return false;
    P.stages = stages;
    P.NB = NB;
    P.family = 4;
    return true;
}

// One cooperative launch of `grid` CTAs in clusters of KS (all CTAs co-resident
// or the launch fails).  If this runtime refuses cooperative cluster launches,
// the cluster launch goes ahead when the occupancy calculator says every
// cluster fits at once (the kernels' waits are bounded either way).
template <class Kern, class Prm>
cudaError_t launch_cluster(Kern kern, const Prm &prm, int grid, int KS, size_t smem,
                           cudaStream_t s, int threads = rec::NUM_THREADS) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = KS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    at[1].id = cudaLaunchAttributeCooperative;
    at[1].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    // Profilers cannot replay a cooperative cluster launch: with
    // LSTM_LAUNCH_NONCOOP=1, or when a profiler or sanitizer is attached, go
    // straight to the occupancy-checked cluster launch below.
    if (!profiler_attached()) {
        e = cudaLaunchKernelEx(&cfg, kern, prm);
        if (e == cudaSuccess || e == cudaErrorCooperativeLaunchTooLarge) {
            note_launch();
            return e;
        }
        cudaGetLastError();
    }
    cfg.numAttrs = 1;  // cluster launch without the cooperative attribute
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess ||
        nclusters * KS < grid) {
        cudaGetLastError();
        return cudaErrorCooperativeLaunchTooLarge;
    }
    note_launch();
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

template <int NB, int KS>
cudaError_t launch_fwd2_t(const rec2::Fwd2Params &prm, const Rec2Plan &P, cudaStream_t s) {
    return launch_cluster(rec2::fwd2_kernel<NB, KS>, prm, P.R * KS * P.G, KS, P.smem, s,
                          rec2::F_THREADS);
}

cudaError_t launch_fwd2(const rec2::Fwd2Params &prm, const Rec2Plan &P, cudaStream_t s) {
#define LSTM_F2(nb, ks) \
    if (P.NB == nb && P.KS == ks) return launch_fwd2_t<nb, ks>(prm, P, s);
    LSTM_F2(16, 1) LSTM_F2(16, 2) LSTM_F2(16, 4)
    LSTM_F2(32, 1) LSTM_F2(32, 2) LSTM_F2(32, 4) LSTM_F2(32, 8)
    LSTM_F2(64, 2) LSTM_F2(64, 4) LSTM_F2(64, 8)
    LSTM_F2(128, 4) LSTM_F2(128, 8)
#undef LSTM_F2
    return cudaErrorInvalidConfiguration;
}

// a2 on the cluster kernel; returns LSTM_ERR_UNSUPPORTED (nothing launched)
// when the plan has no instantiation, so that the caller can fall back.
int tc_fwd_recurrence2(const lstm_dims *d, const Rec2Plan &P, const bf16 *W, const bf16 *h0,
                       const float *c0, const float *Gx, bf16 *y, bf16 *hT, float *cT,
                       bf16 *gates, float *cells, Ctrl *ctrl, cudaStream_t s) {
    const long long T = d->T, B = d->B, H = d->H, I = d->I;
    rec2::Fwd2Params prm;
    memset(&prm, 0, sizeof(prm));
    bool ok = tcg::make_map(&prm.map_w, W, H + I, 4 * H, (H + I) * 2, 64, rec2::F_UNITS) &&
              tcg::make_map(&prm.map_y, y, H, T * B, H * 2, 64, P.NB);
    if (h0) ok = ok && tcg::make_map(&prm.map_h0, h0, H, B, H * 2, 64, P.NB);
    else prm.map_h0 = prm.map_y;
    if (!ok) return LSTM_ERR_UNSUPPORTED;
    prm.Gx = Gx; prm.c0 = c0; prm.y = y; prm.gates = gates; prm.hT = hT;
    prm.cells = cells; prm.cT = cT; prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.R = P.R; prm.G = P.G; prm.kcc = P.kcc;
    prm.has_h0 = h0 != nullptr;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const cudaError_t e = launch_fwd2(prm, P, s);
    if (e == cudaErrorInvalidConfiguration || e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

template <class E, int NB, int KS, int SPLIT>
cudaError_t launch_fwd3_t(const rec3::Fwd3Params<E> &prm, const Rec2Plan &P, cudaStream_t s) {
    if (prm.mask)
        return launch_cluster(rec3::fwd3_kernel<E, NB, KS, true, SPLIT>, prm, P.R * KS * P.G, KS,
                              P.smem, s, rec2::F_THREADS);
    return launch_cluster(rec3::fwd3_kernel<E, NB, KS, false, SPLIT>, prm, P.R * KS * P.G, KS,
                          P.smem, s, rec2::F_THREADS);
}

template <class E>
cudaError_t launch_fwd3(const rec3::Fwd3Params<E> &prm, const Rec2Plan &P, cudaStream_t s) {
#define LSTM_F3(nb, ks) \
    if (P.NB == nb && P.KS == ks) return launch_fwd3_t<E, nb, ks, SPLIT_>(prm, P, s);
    if (P.split == 1) {
        constexpr int SPLIT_ = 1;
        LSTM_F3_SPLIT1(LSTM_F3)
    } else if (P.split == 2) {
        constexpr int SPLIT_ = 2;
        LSTM_F3_SPLIT2(LSTM_F3)
    }
#undef LSTM_F3
    return cudaErrorInvalidConfiguration;
}

// a1 + a2 in one cluster kernel (x-part contracted inside the recurrence);
// LSTM_ERR_NOT_CORESIDENT (nothing launched) lets the caller fall back.
template <class E>
int tc_fwd_recurrence3(const lstm_dims *d, const Rec2Plan &P, const E *x, const E *W,
                       const E *b, const E *h0, const float *c0, const E *mask, bool reverse,
                       bool ijfo, E *y, E *hT, float *cT, E *gates, float *cells, Ctrl *ctrl,
                       cudaStream_t s, int bar_base = 0) {
    const long long T = d->T, B = d->B, H = d->H, I = d->I;
    const CUtensorMapDataType dt = tcg::map_type(Elem<E>::kFmt);
    rec3::Fwd3Params<E> prm;
    memset(&prm, 0, sizeof(prm));
    bool ok = tcg::make_map(&prm.map_y, y, H, T * B, H * 2, 64, P.NB, dt) &&
              tcg::make_map(&prm.map_x, x, I, T * B, I * 2, 64, P.NB, dt);
    if (h0) ok = ok && tcg::make_map(&prm.map_h0, h0, H, B, H * 2, 64, P.NB, dt);
    else prm.map_h0 = prm.map_y;
    if (!ok) return LSTM_ERR_UNSUPPORTED;
    prm.W = W; prm.bias = b; prm.c0 = c0; prm.y = y; prm.gates = gates; prm.hT = hT;
    prm.mask = mask; prm.h0 = h0; prm.reverse = reverse; prm.ijfo = ijfo;
    prm.cells = cells; prm.cT = cT; prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.I = (int)I; prm.R = P.R; prm.G = P.G;
    prm.kcc = P.kcc; prm.kcx = P.kcx;
    prm.has_h0 = h0 != nullptr;
    prm.bar_base = bar_base;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const cudaError_t e = launch_fwd3(prm, P, s);
    if (e == cudaErrorInvalidConfiguration || e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// a3 (+ a5) on the cluster kernel.  W_h^T is written to the workspace first;
// db is the sum of the batch groups' partials.
int tc_bwd_recurrence2(const lstm_dims *d, const Rec2Plan &P, const bf16 *dy, const bf16 *dhT,
                       const float *dcT, const bf16 *W, const float *c0, const bf16 *gates,
                       const float *cells, bf16 *dG, bf16 *WT, float *dbgroup, float *db,
                       float *dh0, float *dc0, Ctrl *ctrl, cudaStream_t s) {
    const long long T = d->T, B = d->B, H = d->H, I = d->I, G4 = 4 * H;
    {
        dim3 grid((unsigned)((H + 31) / 32), (unsigned)((G4 + 31) / 32));
        rec::transpose_wh<<<grid, dim3(32, 8), 0, s>>>(W, WT, (int)H, (int)I);
        note_launch();
        if (cudaGetLastError() != cudaSuccess) return LSTM_ERR_CUDA;
    }
    rec2::Bwd2Params prm;
    memset(&prm, 0, sizeof(prm));
    if (!tcg::make_map(&prm.map_wt, WT, G4, H, G4 * 2, 64, rec2::B_UNITS) ||
        !tcg::make_map(&prm.map_dg, dG, G4, T * B, G4 * 2, 64, P.NB))
        return LSTM_ERR_UNSUPPORTED;
    prm.dy = dy; prm.dhT = dhT; prm.gates = gates; prm.dcT = dcT; prm.cells = cells;
    prm.c0 = c0; prm.dG = dG; prm.dh0 = dh0; prm.dc0 = dc0; prm.db_part = dbgroup;
    prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.U = P.R; prm.G = P.G; prm.NBr = P.NB;
    prm.kcc = P.kcc; prm.stages = P.stages;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const cudaError_t e = launch_cluster(rec2::bwd2_kernel, prm, P.R * P.KS * P.G, P.KS, P.smem, s,
                                         rec2::B_THREADS);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    if (e != cudaSuccess) return LSTM_ERR_CUDA;
    simt::colsum_final<<<(unsigned)((G4 + 255) / 256), 256, 0, s>>>(dbgroup, P.G, (int)G4, db);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// One launch of the TMEM-weight backward kernel over epilogue iterations
// [i0, i1) (time steps T-i1 .. T-i0-1); WT must already hold W_h^T.
template <class E>
int tc_bwd3_launch(const lstm_dims *d, const Rec2Plan &P, const E *dy, const E *dhT,
                   const float *dcT, const float *c0, const E *mask, bool reverse, bool ijfo,
                   const E *gates, const float *cells, E *dG, const E *WT, float *dbgroup,
                   float *dh0, float *dc0, float *dc_carry, float *dhp_carry, Ctrl *ctrl, int i0,
                   int i1, cudaStream_t s, int bar_base = 0) {
    const long long T = d->T, B = d->B, H = d->H, G4 = 4 * H;
    rec3::Bwd3Params<E> prm;
    memset(&prm, 0, sizeof(prm));
    if (!tcg::make_map(&prm.map_dg, dG, G4, T * B, G4 * 2, 64, P.NB,
                       tcg::map_type(Elem<E>::kFmt)))
        return LSTM_ERR_UNSUPPORTED;
    prm.wt = WT;
    prm.dy = dy; prm.dhT = dhT; prm.gates = gates; prm.dcT = dcT; prm.cells = cells;
    prm.c0 = c0; prm.dG = dG; prm.dh0 = dh0; prm.dc0 = dc0; prm.db_part = dbgroup;
    prm.dc_carry = dc_carry;
    prm.mask = mask; prm.dhp_carry = dhp_carry;
    prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.U = P.R; prm.G = P.G; prm.NBr = P.NB;
    prm.kcc = P.kcc; prm.stages = P.stages;
    prm.i0 = i0; prm.i1 = i1; prm.reverse = reverse;
    prm.bar_base = bar_base;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const int nctas = P.R * P.KS * P.G;
    const cudaError_t e =
        mask ? (ijfo ? launch_cluster(rec3::bwd3_kernel<E, true, true>, prm, nctas, P.KS, P.smem,
                                      s, rec3::THREADS)
                     : launch_cluster(rec3::bwd3_kernel<E, true, false>, prm, nctas, P.KS, P.smem,
                                      s, rec3::THREADS))
             : (ijfo ? launch_cluster(rec3::bwd3_kernel<E, false, true>, prm, nctas, P.KS, P.smem,
                                      s, rec3::THREADS)
                     : launch_cluster(rec3::bwd3_kernel<E, false, false>, prm, nctas, P.KS,
                                      P.smem, s, rec3::THREADS));
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// One launch of the two-stream backward kernel over epilogue iterations
// [i0, i1); WT must already hold W_h^T.
template <class E>
int tc_bwd4_launch(const lstm_dims *d, const Rec2Plan &P, const E *dy, const E *dhT,
                   const float *dcT, const float *c0, const E *mask, bool reverse, bool ijfo,
                   const E *gates, const float *cells, E *dG, const E *WT, float *dbgroup,
                   float *dh0, float *dc0, float *dc_carry, float *dhp_carry, Ctrl *ctrl, int i0,
                   int i1, cudaStream_t s, int bar_base = 0) {
    const long long T = d->T, B = d->B, H = d->H, G4 = 4 * H;
    rec4::Bwd4Params<E> prm;
    memset(&prm, 0, sizeof(prm));
    const int NBS = P.NB / rec4::NSTREAM;
    if (!tcg::make_map(&prm.map_dg, dG, G4, T * B, G4 * 2, 64, NBS,
                       tcg::map_type(Elem<E>::kFmt)))
        return LSTM_ERR_UNSUPPORTED;
    prm.wt = WT;
    prm.dy = dy; prm.dhT = dhT; prm.gates = gates; prm.dcT = dcT; prm.cells = cells;
    prm.c0 = c0; prm.dG = dG; prm.dh0 = dh0; prm.dc0 = dc0; prm.db_part = dbgroup;
    prm.dc_carry = dc_carry;
    prm.mask = mask; prm.dhp_carry = dhp_carry;
    prm.ctrl = ctrl;
    prm.T = (int)T; prm.B = (int)B; prm.H = (int)H; prm.U = P.R; prm.G = P.G; prm.NBr = P.NB;
    prm.NBS = NBS; prm.kcc = P.kcc; prm.stages = P.stages;
    prm.i0 = i0; prm.i1 = i1; prm.reverse = reverse;
    prm.bar_base = bar_base;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    const int nctas = P.R * P.KS * P.G;
    const cudaError_t e =
        mask ? (ijfo ? launch_cluster(rec4::bwd4_kernel<E, true, true>, prm, nctas, P.KS, P.smem,
                                      s, rec4::THREADS)
                     : launch_cluster(rec4::bwd4_kernel<E, true, false>, prm, nctas, P.KS, P.smem,
                                      s, rec4::THREADS))
             : (ijfo ? launch_cluster(rec4::bwd4_kernel<E, false, true>, prm, nctas, P.KS, P.smem,
                                      s, rec4::THREADS)
                     : launch_cluster(rec4::bwd4_kernel<E, false, false>, prm, nctas, P.KS,
                                      P.smem, s, rec4::THREADS));
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// One launch of the TMEM-weight backward family the plan names.
template <class E>
int tc_bwd_tmem_launch(const lstm_dims *d, const Rec2Plan &P, const E *dy, const E *dhT,
                       const float *dcT, const float *c0, const E *mask, bool reverse, bool ijfo,
                       const E *gates, const float *cells, E *dG, const E *WT, float *dbgroup,
                       float *dh0, float *dc0, float *dc_carry, float *dhp_carry, Ctrl *ctrl,
                       int i0, int i1, cudaStream_t s, int bar_base = 0) {
    if (P.family == 4)
        return tc_bwd4_launch(d, P, dy, dhT, dcT, c0, mask, reverse, ijfo, gates, cells, dG, WT,
                              dbgroup, dh0, dc0, dc_carry, dhp_carry, ctrl, i0, i1, s, bar_base);
    return tc_bwd3_launch(d, P, dy, dhT, dcT, c0, mask, reverse, ijfo, gates, cells, dG, WT,
                          dbgroup, dh0, dc0, dc_carry, dhp_carry, ctrl, i0, i1, s, bar_base);
}

// W_h^T of a 16-bit W (bf16 or fp16: the kernels only move 16-bit values):
// 64 x 64 tiles with 16-byte accesses when the rows allow, else 32 x 32 tiles
// of single elements.
cudaError_t launch_transpose_wh(const lstm_dims *d, const void *W_, void *WT_, cudaStream_t s) {
    const long long H = d->H, I = d->I, G4 = 4 * H;
    if (H % 8 == 0 && I % 8 == 0 && aligned16(W_) && aligned16(WT_)) {
        dim3 grid((unsigned)((H + 63) / 64), (unsigned)((G4 + 63) / 64));
        rec::transpose_wh_v8<<<grid, 256, 0, s>>>(static_cast<const uint16_t *>(W_),
                                                   static_cast<uint16_t *>(WT_), (int)H, (int)I);
        note_launch();
        return cudaGetLastError();
    }
    const bf16 *W = static_cast<const bf16 *>(W_);
    bf16 *WT = static_cast<bf16 *>(WT_);
    dim3 grid((unsigned)((H + 31) / 32), (unsigned)((G4 + 31) / 32));
    rec::transpose_wh<<<grid, dim3(32, 8), 0, s>>>(W, WT, (int)H, (int)d->I);
    note_launch();
    return cudaGetLastError();
}

// a3 (+ a5) on the cluster kernel with W_h^T in TMEM (written to the
// workspace first, then copied into each CTA's tensor memory), one launch.
template <class E>
int tc_bwd_recurrence3(const lstm_dims *d, const Rec2Plan &P, const E *dy, const E *dhT,
                       const float *dcT, const E *W, const float *c0, const E *mask,
                       bool reverse, bool ijfo, const E *gates, const float *cells, E *dG,
                       E *WT,
                       float *dbgroup, float *db, float *dh0, float *dc0, Ctrl *ctrl,
                       cudaStream_t s) {
    const long long G4 = 4LL * d->H;
    if (launch_transpose_wh(d, W, WT, s) != cudaSuccess) return LSTM_ERR_CUDA;
    const int rc = tc_bwd_tmem_launch(d, P, dy, dhT, dcT, c0, mask, reverse, ijfo, gates, cells,
                                      dG, WT, dbgroup, dh0, dc0, nullptr, nullptr, ctrl, 0, d->T,
                                      s);
    if (rc != LSTM_OK) return rc;
    simt::colsum_final<<<(unsigned)((G4 + 255) / 256), 256, 0, s>>>(dbgroup, P.G, (int)G4, db);
    note_launch();
    return cudaGetLastError() == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// One warp that returns `ns` nanoseconds after it starts (at most 2^20 naps
// of 256 ns).  In a stream before a GEMM that becomes ready at the moment the
// next launch of a persistent cluster kernel does, it lets that launch take
// its SMs first: a GEMM placed CTA by CTA on the SMs just freed can break up
// the cluster slots the launch needs, which then waits for the GEMM to end.
// It touches no memory and needs so few resources that it fits beside any
// resident kernel, so it never holds an SM that launch needs.
__global__ void __launch_bounds__(32, 1) hold_ns(unsigned long long ns) {
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (int i = 0; i < (1 << 20); ++i) {
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 >= ns) break;
        __nanosleep(256);
    }
}
constexpr unsigned long long kGemmHoldNs = 8000;

cudaError_t launch_hold(cudaStream_t s) {
    hold_ns<<<1, 32, 0, s>>>(kGemmHoldNs);
    note_launch();
    return cudaGetLastError();
}

// a3 + a5 in `nch` reverse-time chunks (one launch each, delta c carried
// through the workspace) on a high-priority stream, and a4 + a6 of every
// finished chunk on a low-priority stream, beside the next chunk: the GEMM
// takes the SMs the recurrence leaves idle (all of them for the last chunk).
// No kernel waits on another; the streams are ordered by events and joined
// back into `s` on every return.
template <class E>
int tc_bwd3_overlapped(const lstm_dims *d, const Rec2Plan &P, AuxStreams &A, int nch,
                       const E *dy, const E *dhT, const float *dcT, const E *x,
                       const E *W, const E *h0, const float *c0, const E *mask,
                       bool reverse, bool ijfo, const E *y, const E *gates,
                       const float *cells,
                       E *dG, E *WT, float *dbgroup, float *dc_carry, float *dhp_carry,
                       float *dx, float *dW, float *db, float *dh0, float *dc0, Ctrl *ctrl,
                       cudaStream_t s) {
    std::lock_guard<std::mutex> lock(A.mu);
    const int T = d->T;
    const long long G4 = 4LL * d->H;
    cudaEvent_t ev_fork = A.ev[kMaxChunks], ev_rec = A.ev[kMaxChunks + 1],
                ev_gemm = A.ev[kMaxChunks + 2];
    if (cudaEventRecord(ev_fork, s) != cudaSuccess ||
        cudaStreamWaitEvent(A.rec, ev_fork, 0) != cudaSuccess ||
        cudaStreamWaitEvent(A.gemm, ev_fork, 0) != cudaSuccess)
        return LSTM_ERR_CUDA;
    // the GEMM beside the recurrence takes at most the SMs the recurrence
    // leaves idle
    const int gemm_ctas = std::max(1, tcg::sm_count() - P.R * P.KS * P.G);
    int rc = LSTM_OK;
    {
        prof::Phase ph(LSTM_PHASE_BWD_RECUR, A.rec);
        if (launch_transpose_wh(d, W, WT, A.rec) != cudaSuccess) rc = LSTM_ERR_CUDA;
        for (int c = 0; c < nch && rc == LSTM_OK; ++c) {
            const int i0 = chunk_bound(T, nch, c), i1 = chunk_bound(T, nch, c + 1);
            rc = tc_bwd_tmem_launch(d, P, dy, dhT, dcT, c0, mask, reverse, ijfo, gates, cells, dG,
                                    WT, dbgroup, dh0, dc0, dc_carry, dhp_carry, ctrl, i0, i1,
                                    A.rec);
            if (rc != LSTM_OK) break;
            if (cudaEventRecord(A.ev[c], A.rec) != cudaSuccess ||
                cudaStreamWaitEvent(A.gemm, A.ev[c], 0) != cudaSuccess ||
                (c + 1 < nch && launch_hold(A.gemm) != cudaSuccess)) {
                rc = LSTM_ERR_CUDA;
                break;
            }
            prof::Phase phg(LSTM_PHASE_DW, A.gemm);
            // rows of the chunk's times (steps T-i1 .. T-i0-1: times i0 .. i1-1 in
            // the reverse direction); dW accumulates after the first chunk
            const int t_lo = reverse ? i0 : T - i1, t_hi = reverse ? i1 : T - i0;
            if (tc_dw_dx(d, dG, x, W, h0, y, dW, dx, ctrl, A.gemm, t_lo, t_hi, c > 0,
                         c + 1 < nch ? gemm_ctas : 0, reverse) != cudaSuccess)
                rc = LSTM_ERR_CUDA;
        }
        if (rc == LSTM_OK) {
            simt::colsum_final<<<(unsigned)((G4 + 255) / 256), 256, 0, A.rec>>>(dbgroup, P.G,
                                                                                 (int)G4, db);
            note_launch();
            if (cudaGetLastError() != cudaSuccess) rc = LSTM_ERR_CUDA;
        }
    }
    // join: nothing of this call stays unordered with the caller's stream
    if (cudaEventRecord(ev_rec, A.rec) != cudaSuccess ||
        cudaEventRecord(ev_gemm, A.gemm) != cudaSuccess ||
        cudaStreamWaitEvent(s, ev_rec, 0) != cudaSuccess ||
        cudaStreamWaitEvent(s, ev_gemm, 0) != cudaSuccess)
        return LSTM_ERR_CUDA;
    return rc;
}

// --------------------------------- persistent CUDA-core recurrences (pst)
// One cooperative launch of `grid` CTAs of pst::NTHR threads (all co-resident
// or nothing runs); with a profiler attached, an occupancy-checked plain launch.
template <class Kern, class Prm>
cudaError_t launch_persistent(Kern kern, const Prm &prm, int grid, size_t smem, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, pst::NTHR, smem) != cudaSuccess ||
        per_sm * tcg::sm_count() < grid) {
        cudaGetLastError();
        return cudaErrorCooperativeLaunchTooLarge;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(pst::NTHR);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    cfg.attrs = at;
    cfg.numAttrs = profiler_attached() ? 0 : 1;
    note_launch();
    return cudaLaunchKernelEx(&cfg, kern, prm);
}

// Whether `grid` CTAs of `kern` in clusters of KS (1: no clusters) can all be
// resident at once with `smem` bytes of dynamic shared memory each.
template <class Kern>
bool pst_coresident(Kern kern, int KS, int grid, size_t smem) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    if (KS == 1) {
        int per_sm = 0;
        const bool ok = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, pst::NTHR,
                                                                      smem) == cudaSuccess &&
                        per_sm * tcg::sm_count() >= grid;
        cudaGetLastError();
        return ok;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(pst::NTHR);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = KS;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nclusters = 0;
    const bool ok = cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) == cudaSuccess &&
                    nclusters * KS >= grid;
    cudaGetLastError();
    return ok;
}

// Work split of the persistent recurrences (pst::Split): for each cluster
// size KS in 8, 4, 2, 1 the fewest units per CTA (quads in the backward, the
// grain of its epilogue) that keep the grid within one CTA per SM and
// co-resident (more units per CTA, fewer clusters, while it is not), the
// staging chunk (at most 16384 floats over all B rows, halved until the
// shared memory fits) and the lanes per dot product (those the CTA would
// otherwise leave idle); of the splits that fit and are co-resident, the one
// with the lowest estimated step time in SM cycles: the K slice's operand
// bytes at 16 B per cycle (an SM's share of L2 in the burst after a step
// barrier), the exchange (≈ 1200 cycles plus its bytes at the same rate), the
// contraction (≈ 42 cycles per float4 column step of a thread's items: two
// warps per scheduler, ≈ 21 instructions each) and 300 cycles per extra chunk.
// LSTM_PERSIST_KS=n keeps only cluster size n.
struct PstPlan {
    pst::Split s = {};
    int P = 0;
    size_t smem = 0;
};
int g_last_pst_ks[2] = {0, 0};  // cluster size of the last persistent fwd / bwd (test hook)

template <class T>
bool plan_persist(const lstm_dims *d, bool backward, PstPlan &Q) {
    if (env_is("LSTM_PERSIST", '0') || d->H < 1 || d->B < 1 || d->T < 1) return false;
    const char *ov = getenv("LSTM_PERSIST_KS");
    const int only = ov ? atoi(ov) : 0;
    const int nsm = tcg::sm_count(), B = d->B, H = d->H;
    const int q = backward ? 4 : 1;
    const int K = backward ? 4 * H : H;
    double best = 1e30;
    for (int KS : {8, 4, 2, 1}) {
        if (only && only != KS) continue;
        pst::Split s = {};
        s.KS = KS;
        s.KSL = ((K + KS - 1) / KS + 7) / 8 * 8;
        if (KS > 1 && (long long)s.KSL * (KS - 1) >= K) continue;  // a rank without columns
        s.UN = q;
        while ((long long)(H + KS * s.UN - 1) / (KS * s.UN) * KS > nsm) s.UN += q;
        // more units per CTA (fewer clusters) until the grid is co-resident
        int UC = 0, P = 0;
        long long items = 0;
        size_t smem = 0;
        bool fits = false;
        for (; !fits; s.UN += q) {
            UC = KS * s.UN;
            P = (H + UC - 1) / UC * KS;
            items = (long long)B * (backward ? UC / 4 : UC);
            if (items > (long long)pst::MAXP * pst::NTHR) break;
            s.KSPLIT = 1;
            while (s.KSPLIT < 32 && items * s.KSPLIT * 2 <= pst::NTHR) s.KSPLIT *= 2;
            const int pad = 4 * std::min(s.KSPLIT, 8);
            s.KC = std::min(std::max(32, 16384 / B / 32 * 32), (s.KSL + 31) / 32 * 32);
            s.KCP = s.KC + pad;
            while (s.KC > 32 && pst::layout(backward, B, s).bytes > kMaxSmem) {
                s.KC = std::max(32, s.KC / 2 / 32 * 32);
                s.KCP = s.KC + pad;
            }
            smem = pst::layout(backward, B, s).bytes;
            if (smem > kMaxSmem) break;
            fits = backward ? pst_coresident(pst::bwd_kernel<T>, KS, P, smem)
                            : pst_coresident(pst::fwd_kernel<T>, KS, P, smem);
            if (fits) break;
        }
        if (!fits) continue;
        const int nslots = pst::NTHR / s.KSPLIT;
        const double cost =
            (double)B * s.KSL * sizeof(T) / 16.0 +
            (KS > 1 ? 1200.0 + (KS - 1) * pst::part_floats(backward, B, s.UN) * 4 / 16.0 : 0.0) +
            42.0 * (double)((items + nslots - 1) / nslots) *
                (double)((s.KSL / 4 + s.KSPLIT - 1) / s.KSPLIT) +
            300.0 * (double)((s.KSL + s.KC - 1) / s.KC - 1);
        if (cost < best) {
            best = cost;
            Q.s = s;
            Q.P = P;
            Q.smem = smem;
        }
    }
    return best < 1e30;
}

// One launch of a persistent recurrence: a cooperative cluster launch when the
// split has KS > 1.  LSTM_ERR_NOT_CORESIDENT (nothing launched) lets the
// caller fall back.
template <class Kern, class Prm>
int launch_pst(Kern kern, const Prm &prm, const PstPlan &Q, cudaStream_t s) {
    const cudaError_t e = Q.s.KS > 1
                              ? launch_cluster(kern, prm, Q.P, Q.s.KS, Q.smem, s, pst::NTHR)
                              : launch_persistent(kern, prm, Q.P, Q.smem, s);
    if (e == cudaErrorCooperativeLaunchTooLarge) {
        cudaGetLastError();
        return LSTM_ERR_NOT_CORESIDENT;
    }
    return e == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

// a2 over all T steps in one launch; Gx holds the input projection.
template <class T>
int persist_fwd(const lstm_dims *d, const PstPlan &Q, const T *W, const float *Gx,
                const T *h0, const float *c0, const T *mask, bool reverse, bool ijfo, T *y,
                T *gates, float *cells, Ctrl *ctrl, cudaStream_t s) {
    pst::FwdParams<T> prm;
    memset(&prm, 0, sizeof(prm));
    prm.W = W; prm.Gx = Gx; prm.h0 = h0; prm.c0 = c0; prm.mask = mask;
    prm.y = y; prm.gates = gates; prm.cells = cells; prm.ctrl = ctrl;
    prm.T = d->T; prm.B = d->B; prm.H = d->H; prm.I = d->I;
    prm.reverse = reverse; prm.fb = ijfo ? 2 : 1;
    prm.s = Q.s;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    g_last_pst_ks[0] = Q.s.KS;
    return launch_pst(pst::fwd_kernel<T>, prm, Q, s);
}

// a3 over all T steps in one launch, and dinitH = W_h^T dG of the first step
// as one more contraction at its end.
template <class T>
int persist_bwd(const lstm_dims *d, const PstPlan &Q, const T *W, const T *dy,
                const T *dhT, const float *dcT, const T *gates, const float *cells,
                const float *c0, const T *mask, bool reverse, bool ijfo, T *dG,
                float *const dcbuf[2], float *const dhpbuf[2], float *dc0, float *dh0,
                Ctrl *ctrl, cudaStream_t s) {
    pst::BwdParams<T> prm;
    memset(&prm, 0, sizeof(prm));
    prm.W = W; prm.dy = dy; prm.dhT = dhT; prm.gates = gates; prm.mask = mask;
    prm.dcT = dcT; prm.cells = cells; prm.c0 = c0; prm.dG = dG;
    prm.dcbuf[0] = dcbuf[0]; prm.dcbuf[1] = dcbuf[1];
    prm.dhpbuf[0] = dhpbuf[0]; prm.dhpbuf[1] = dhpbuf[1];
    prm.dc0 = dc0; prm.dh0 = dh0; prm.ctrl = ctrl;
    prm.T = d->T; prm.B = d->B; prm.H = d->H; prm.I = d->I;
    prm.reverse = reverse; prm.fb = ijfo ? 2 : 1;
    prm.s = Q.s;
    prm.fault_skip_cta = g_fault_skip_cta;
    prm.wait_ns = g_wait_ns;
    g_last_pst_ks[1] = Q.s.KS;
    return launch_pst(pst::bwd_kernel<T>, prm, Q, s);
}

// ------------------------------------------------------------ forward pass
// mask (variable length) or NULL; masked calls run on the TMEM-weight cluster
// kernel or the per-step kernels only.
// plan3: the fused forward's plan when it applies (NULL otherwise); every
// other path needs the Gx buffer, i.e. ws_bytes >= fwd_layout(d).total.
template <class T>
int fwd_simt(const lstm_dims *d, const T *x, const T *W, const T *b, const T *h0,
             const float *c0, const T *mask, bool reverse, bool ijfo, T *y, T *hT, float *cT,
             T *gates, float *cells, char *ws, size_t ws_bytes, const Rec2Plan *plan3,
             cudaStream_t s) {
    typedef typename Tc16<T>::type E;  // the 16-bit type of the tensor-core paths
    // masked, reverse-direction, "ijfo" or fp16 calls: TMEM-weight kernel or
    // per-step kernels (the other kernels are bf16 / default-order only)
    const bool special = mask != nullptr || reverse || ijfo || d->dtype == LSTM_F16;
    const int T_ = d->T, B = d->B, I = d->I, H = d->H;
    const long long BH = (long long)B * H;
    const FwdLayout L = fwd_layout(d);
    float *Gx = (float *)(ws + L.gx);
    if ((long long)T_ * B > 0 && H > 0) {
        if (plan3) {  // a1 fused into a2
            prof::Phase ph(LSTM_PHASE_FWD_RECUR, s);
            const int rc = tc_fwd_recurrence3(d, *plan3, (const E *)x, (const E *)W,
                                              (const E *)b, (const E *)h0, c0,
                                              (const E *)mask, reverse, ijfo, (E *)y,
                                              (E *)hT, cT, (E *)gates, cells,
                                              (Ctrl *)ws, s);
            g_last_fwd_path = 3;
            if (rc != LSTM_ERR_NOT_CORESIDENT) return rc;
        }
        // every path below reads the input projection from Gx
        if (ws_bytes < L.total) return LSTM_ERR_WORKSPACE;
        {   // a1: Gx = X W_x^T + b over all T*B rows (input concat, x-part)
            prof::Phase ph(LSTM_PHASE_INPUT_PROJ, s);
            if (tc_gemm_ok(d)) {
                LSTM_TRY(tc_input_projection(d, (const E *)x,
                                             (const E *)W,
                                             (const E *)b, Gx, (Ctrl *)ws, s));
            } else {
                LSTM_TRY((simt::gemm<true, true>(T_ * B, 4 * H, I, simt::RowMajor<T>{x, I},
                                                  simt::WxT<T>{W, H, I},
                                                  simt::EpGx<T>{Gx, b, 4 * H}, s)));
            }
        }
        // a2: the recurrence
        prof::Phase ph(LSTM_PHASE_FWD_RECUR, s);
        Rec2Plan plan2;
        if (!special && plan_fwd2(d, plan2)) {
            const int rc = tc_fwd_recurrence2(d, plan2, (const bf16 *)W, (const bf16 *)h0, c0, Gx,
                                              (bf16 *)y, (bf16 *)hT, cT, (bf16 *)gates, cells,
                                              (Ctrl *)ws, s);
            g_last_fwd_path = 2;
            if (rc != LSTM_ERR_NOT_CORESIDENT) return rc;
        }
        RecPlan plan;
        if (!special && plan_fwd_recur(d, plan)) {
            g_last_fwd_path = 1;
            // persistent tcgen05 kernel: all T steps in one launch; it writes hT and cT
            return tc_fwd_recurrence(d, plan, (const bf16 *)W, (const bf16 *)h0, c0, Gx,
                                     (bf16 *)y, (bf16 *)hT, cT, (bf16 *)gates, cells, (Ctrl *)ws,
                                     s);
        }
        // otherwise the persistent CUDA-core recurrence (all steps, one launch)
        bool persisted = false;
        {
            PstPlan Q;
            if (plan_persist<T>(d, false, Q)) {
                const int rc = persist_fwd<T>(d, Q, W, Gx, h0, c0, mask, reverse, ijfo,
                                              y, gates, cells, (Ctrl *)ws, s);
                if (rc != LSTM_ERR_NOT_CORESIDENT && rc != LSTM_OK) return rc;
                persisted = rc == LSTM_OK;
            }
        }
        // or one fused GEMM + gate/cell/hidden epilogue launch per step
        g_last_fwd_path = persisted ? 5 : 0;
        for (int st = 0; !persisted && st < T_; ++st) {
            // step st is at time t; the previous step at time tp
            const int t = reverse ? T_ - 1 - st : st, tp = reverse ? t + 1 : t - 1;
            const T *hp = st > 0 ? y + (long long)tp * BH : h0;
            const float *cp = st > 0 ? cells + (long long)tp * BH : c0;
            simt::EpFwdStep<T> ep{Gx + (long long)t * B * 4 * H, cp, y + (long long)t * BH,
                                  gates + (long long)t * B * 4 * H, cells + (long long)t * BH, H};
            if (mask) {
                ep.mask = mask + (long long)t * BH;
                ep.hprev = hp;
            }
            ep.fb = ijfo ? 2 : 1;
            LSTM_TRY((simt::gemm<true, true>(B, 4 * H, H, simt::Hprev<T>{hp, H},
                                              simt::WhT4<T>{W, H, I}, ep, s)));
        }
    }
    if (BH > 0) {
        prof::Phase ph(LSTM_PHASE_OTHER, s);
        if (T_ > 0) {  // the state after the last step (time 0 in the reverse direction)
            const long long tl = reverse ? 0 : T_ - 1;
            LSTM_TRY(cudaMemcpyAsync(hT, y + tl * BH, BH * sizeof(T), cudaMemcpyDeviceToDevice,
                                     s));
            LSTM_TRY(cudaMemcpyAsync(cT, cells + tl * BH, BH * sizeof(float),
                                     cudaMemcpyDeviceToDevice, s));
        } else {
            LSTM_TRY(launch_copy_or_zero<T>(h0, hT, BH, s));
            LSTM_TRY(launch_copy_or_zero<float>(c0, cT, BH, s));
        }
    }
    return LSTM_OK;
}

// ----------------------------------------------------------- backward pass
// mask (variable length) or NULL; masked calls run on the TMEM-weight cluster
// kernel or the per-step kernels only.
template <class T>
int bwd_simt(const lstm_dims *d, const T *dy, const T *dhT, const float *dcT, const T *x,
             const T *W, const T *h0, const float *c0, const T *mask, bool reverse, bool ijfo,
             const T *y, const T *gates, const float *cells, float *dx, float *dW, float *db,
             float *dh0, float *dc0, char *ws, cudaStream_t s) {
    typedef typename Tc16<T>::type E;  // the 16-bit type of the tensor-core paths
    const bool special = mask != nullptr || reverse || ijfo || d->dtype == LSTM_F16;
    const int T_ = d->T, B = d->B, I = d->I, H = d->H;
    const long long BH = (long long)B * H, TB = (long long)T_ * B;
    const int G4 = 4 * H, K = H + I;
    const BwdLayout L = bwd_layout(d);
    T *dG = (T *)(ws + L.dG);
    float *dcbuf[2] = {(float *)(ws + L.dc), (float *)(ws + L.dc) + BH};
    float *dhpbuf[2] = {(float *)(ws + L.dhp), (float *)(ws + L.dhp) + BH};

    if (TB == 0 || H == 0) {
        // no step runs: the incoming gradients pass straight through
        prof::Phase ph(LSTM_PHASE_OTHER, s);
        LSTM_TRY(launch_to_float<T>(T_ == 0 ? dhT : nullptr, dh0, BH, s));
        LSTM_TRY(launch_copy_or_zero<float>(T_ == 0 ? dcT : nullptr, dc0, BH, s));
        if ((long long)G4 * K > 0) LSTM_TRY(cudaMemsetAsync(dW, 0, (size_t)G4 * K * sizeof(float), s));
        if (G4 > 0) LSTM_TRY(cudaMemsetAsync(db, 0, (size_t)G4 * sizeof(float), s));
        if (TB * I > 0) LSTM_TRY(cudaMemsetAsync(dx, 0, (size_t)(TB * I) * sizeof(float), s));
        return LSTM_OK;
    }

    RecPlan plan;
    Rec2Plan plan2, plan3;
    const bool v3 = plan_bwd4(d, plan3) || plan_bwd3(d, plan3);
    const bool v2 = !v3 && !special && plan_bwd2(d, plan2);
    const bool v1 = !special && plan_bwd_recur(d, plan);
    bool per_step = false;  // a special call whose cluster kernel cannot be placed
    if (v3 || v2 || v1) {
        if (v3 && tc_gemm_ok(d) && bwd_chunks(d) > 1) {
            AuxStreams *A = aux_streams();
            if (A) {  // a3 + a5 with a4 + a6 overlapped
                g_last_bwd_path = plan3.family;
                const int rc = tc_bwd3_overlapped(
                    d, plan3, *A, bwd_chunks(d), (const E *)dy, (const E *)dhT, dcT,
                    (const E *)x, (const E *)W, (const E *)h0, c0, (const E *)mask,
                    reverse, ijfo, (const E *)y, (const E *)gates, cells, (E *)dG,
                    (E *)(ws + L.wt), (float *)(ws + L.dbgroup), (float *)(ws + L.dc),
                    (float *)(ws + L.dhp), dx, dW, db, dh0, dc0, (Ctrl *)ws, s);
                if (rc != LSTM_ERR_NOT_CORESIDENT) return rc;
            }
        }
        {   // a3 + a5: persistent tcgen05 recurrence with db fused
            prof::Phase ph(LSTM_PHASE_BWD_RECUR, s);
            int rc = LSTM_ERR_NOT_CORESIDENT;
            g_last_bwd_path = v3 ? plan3.family : 2;
            if (v3)
                rc = tc_bwd_recurrence3(d, plan3, (const E *)dy, (const E *)dhT, dcT,
                                        (const E *)W, c0, (const E *)mask, reverse, ijfo,
                                        (const E *)gates, cells, (E *)dG,
                                        (E *)(ws + L.wt), (float *)(ws + L.dbgroup), db, dh0,
                                        dc0, (Ctrl *)ws, s);
            else if (v2)
                rc = tc_bwd_recurrence2(d, plan2, (const bf16 *)dy, (const bf16 *)dhT, dcT,
                                        (const bf16 *)W, c0, (const bf16 *)gates, cells,
                                        (bf16 *)dG, (bf16 *)(ws + L.wt),
                                        (float *)(ws + L.dbgroup), db, dh0, dc0, (Ctrl *)ws, s);
            if (rc == LSTM_ERR_NOT_CORESIDENT && v1) {
                g_last_bwd_path = 1;
                rc = tc_bwd_recurrence(
                d, plan, (const bf16 *)dy, (const bf16 *)dhT, dcT, (const bf16 *)W, c0,
                (const bf16 *)gates, cells, (bf16 *)dG, (bf16 *)(ws + L.wt),
                (float *)(ws + L.dbgroup), db, dh0, dc0, (Ctrl *)ws, s);
            }
            if (rc == LSTM_ERR_NOT_CORESIDENT && special) per_step = true;
            else if (rc != LSTM_OK) return rc;
        }
        if (!per_step) {
            if (tc_gemm_ok(d)) {
                prof::Phase ph(LSTM_PHASE_DW, s);
                LSTM_TRY(tc_dw_dx(d, (const E *)dG, (const E *)x, (const E *)W,
                                  (const E *)h0, (const E *)y, dW, dx, (Ctrl *)ws, s, 0,
                                  d->T, false, 0, reverse));
                return LSTM_OK;
            }
            // dW / dx on CUDA cores (shapes off the TMA grid)
            {
                prof::Phase ph(LSTM_PHASE_DW, s);
                LSTM_TRY((simt::gemm<false, false>(G4, K, (int)TB, simt::ColMajor<T>{dG, G4},
                                                    simt::Zrows<T>{x, y, h0, B, I, H, reverse, (long long)(T_ - 1) * B},
                                                    simt::EpStore{dW, K}, s)));
            }
            prof::Phase ph(LSTM_PHASE_DX, s);
            if (I > 0)
                LSTM_TRY((simt::gemm<true, false>((int)TB, I, G4, simt::RowMajor<T>{dG, G4},
                                                   simt::RowMajor<T>{W + H, K},
                                                   simt::EpStore{dx, I}, s)));
            return LSTM_OK;
        }
    }

    // a3: reverse-time recursion, steps 1-3 and 5 fused with delta h = W_h^T dG_{t+1}:
    // the persistent CUDA-core recurrence (all steps, one launch), or one launch per step
    {
    prof::Phase ph(LSTM_PHASE_BWD_RECUR, s);
    bool persisted = false;
    {
        PstPlan Q;
        if (plan_persist<T>(d, true, Q)) {
            const int rc = persist_bwd<T>(d, Q, W, dy, dhT, dcT, gates, cells, c0, mask,
                                          reverse, ijfo, dG, dcbuf, dhpbuf, dc0, dh0,
                                          (Ctrl *)ws, s);
            if (rc != LSTM_ERR_NOT_CORESIDENT && rc != LSTM_OK) return rc;
            persisted = rc == LSTM_OK;
        }
    }
    g_last_bwd_path = persisted ? 5 : 0;
    // steps st = T-1 .. 0 of the forward recurrence; step st is at time tau(st)
    auto tau = [&](int st) -> long long { return reverse ? T_ - 1 - st : st; };
    for (int st = T_ - 1; !persisted && st >= 0; --st) {
        const bool last = (st == T_ - 1);
        const long long t = tau(st);
        simt::EpBwdStep<T> ep;
        ep.dy = dy ? dy + t * BH : nullptr;
        ep.dh_in = last ? dhT : nullptr;
        ep.dc_in = last ? dcT : dcbuf[(st + 1) & 1];
        ep.gates = gates + t * B * G4;
        ep.cells = cells + t * BH;
        ep.cprev = st > 0 ? cells + tau(st - 1) * BH : c0;
        ep.dG = dG + t * B * G4;
        ep.dc_out = (st == 0) ? dc0 : dcbuf[st & 1];
        ep.H = H;
        ep.use_acc = !last;
        ep.fb = ijfo ? 2 : 1;
        if (mask) {
            ep.mask = mask + t * BH;
            ep.dhp_in = last ? nullptr : dhpbuf[(st + 1) & 1];
            ep.dhp_out = dhpbuf[st & 1];
        }
        const T *dGn = last ? dG : dG + tau(st + 1) * B * G4;
        LSTM_TRY((simt::gemm<true, false>(B, H, last ? 0 : G4, simt::RowMajor<T>{dGn, G4},
                                           simt::RowMajor<T>{W, K}, ep, s)));
    }
    // dinitH = W_h^T dG of the first step (delta h_prev before it, step 5), plus
    // what padding at that step passes on (inside the persistent kernel when it ran)
    if (!persisted)
        LSTM_TRY((simt::gemm<true, false>(B, H, G4, simt::RowMajor<T>{dG + tau(0) * B * G4, G4},
                                           simt::RowMajor<T>{W, K},
                                           simt::EpStore{dh0, H, mask ? dhpbuf[0] : nullptr}, s)));
    }
    const bool tc = tc_gemm_ok(d);
    // a4, a5 and a6 only read the finished dG: dW (with dx on the tensor cores)
    // on the caller's stream, db and the CUDA-core dx beside it on the two
    // auxiliary streams when they exist, joined back with events
    AuxStreams *A = aux_streams();
    std::unique_lock<std::mutex> lk;
    if (A) lk = std::unique_lock<std::mutex>(A->mu);
    cudaStream_t s_db = A ? A->rec : s, s_dx = A ? A->gemm : s;
    if (A) {
        LSTM_TRY(cudaEventRecord(A->ev[0], s));
        LSTM_TRY(cudaStreamWaitEvent(s_db, A->ev[0], 0));
        LSTM_TRY(cudaStreamWaitEvent(s_dx, A->ev[0], 0));
    }
    // a5: db = column sums of dG (step 4)
    {
        prof::Phase ph(LSTM_PHASE_DB, s_db);
        float *part = (float *)(ws + L.dbpart);
        dim3 g1((G4 + 255) / 256, L.db_chunks);
        simt::colsum_partial<T><<<g1, 256, 0, s_db>>>(dG, (int)TB, G4, L.db_rows_per_chunk, part);
        note_launch();
        LSTM_TRY(cudaGetLastError());
        simt::colsum_final<<<(G4 + 255) / 256, 256, 0, s_db>>>(part, L.db_chunks, G4, db);
        note_launch();
        LSTM_TRY(cudaGetLastError());
    }
    // a6: dx = dG W_x (x-part of delta z, step 5)
    if (I > 0 && !tc) {
        prof::Phase ph(LSTM_PHASE_DX, s_dx);
        LSTM_TRY((simt::gemm<true, false>((int)TB, I, G4, simt::RowMajor<T>{dG, G4},
                                           simt::RowMajor<T>{W + H, K},
                                           simt::EpStore{dx, I}, s_dx)));
    }
    if (tc) {
        // a4 + a6 together on the tensor cores (one launch, timed as dW)
        prof::Phase ph(LSTM_PHASE_DW, s);
        LSTM_TRY(tc_dw_dx(d, (const E *)dG, (const E *)x, (const E *)W,
                          (const E *)h0, (const E *)y, dW, dx, (Ctrl *)ws, s, 0, d->T,
                          false, 0, reverse));
    } else if (L.dw_splits > 1) {
        // a4: dW = dG^T [h_prev | x] over all T*B rows (step 4), the rows split
        // into dw_splits slabs whose partial products are summed in order
        prof::Phase ph(LSTM_PHASE_DW, s);
        float *part = (float *)(ws + L.dwsplit);
        const long long MN = G4 * K;
        LSTM_TRY((simt::gemm<false, false>(G4, K, (int)TB, simt::ColMajor<T>{dG, G4},
                                            simt::Zrows<T>{x, y, h0, B, I, H, reverse, (long long)(T_ - 1) * B},
                                            simt::EpPart{part, (int)K, MN}, s, L.dw_splits)));
        simt::sum_splits<<<(unsigned)((MN + 255) / 256), 256, 0, s>>>(part, L.dw_splits, MN, dW);
        note_launch();
        LSTM_TRY(cudaGetLastError());
    } else {
        // a4: dW = dG^T [h_prev | x] over all T*B rows (step 4)
        prof::Phase ph(LSTM_PHASE_DW, s);
        LSTM_TRY((simt::gemm<false, false>(G4, K, (int)TB, simt::ColMajor<T>{dG, G4},
                                            simt::Zrows<T>{x, y, h0, B, I, H, reverse, (long long)(T_ - 1) * B},
                                            simt::EpStore{dW, K}, s)));
    }
    if (A) {
        LSTM_TRY(cudaEventRecord(A->ev[1], s_db));
        LSTM_TRY(cudaEventRecord(A->ev[2], s_dx));
        LSTM_TRY(cudaStreamWaitEvent(s, A->ev[1], 0));
        LSTM_TRY(cudaStreamWaitEvent(s, A->ev[2], 0));
    }
    return LSTM_OK;
}

}  // namespace

namespace {
// The forward's plan on the current device: the fused kernel (input projection
// inside the recurrence) when it applies to these dims and options.
bool fwd_fused_plan(const lstm_dims *d, bool masked, Rec2Plan &P) {
    return (long long)d->T * d->B > 0 && d->H > 0 && plan_fwd3(d, P, masked);
}

// Bytes the forward needs: the 256-byte control block alone when the fused
// kernel runs, else the control block and the fp32 Gx buffer.
size_t fwd_ws_need(const lstm_dims *d, bool masked) {
    Rec2Plan P;
    return fwd_fused_plan(d, masked, P) ? kCtrlBytes : fwd_layout(d).total;
}
}  // namespace

// ------------------------------------------ scratch for lstm_fwd_noalloc
// A file-scope device array: every GPU that loads this library holds
// LSTM_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host code the
// name g_noalloc_scratch is only a host-side stand-in for the symbol, never a
// device address; the address is looked up per device below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LSTM_NOALLOC_SCRATCH_BYTES];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current) and cached.
int noalloc_scratch(void **out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return LSTM_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LSTM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LSTM_ERR_CUDA;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LSTM_OK;
}
}  // namespace

// =================================================================== C ABI
namespace {
int fwd_entry(const lstm_dims *d, const lstm_options *opt, const void *x, const void *W,
              const void *b, const void *h0, const float *c0, void *y, void *hT, float *cT,
              void *gates, float *cells, void *ws, size_t ws_bytes, void *stream) {
    if (!dims_ok(d)) return LSTM_ERR_INVALID_ARG;
    const void *mask = opt ? opt->seq_mask : nullptr;
    const int dir = opt ? opt->direction : LSTM_DIR_FORWARD;
    if (dir != LSTM_DIR_FORWARD && dir != LSTM_DIR_REVERSE) return LSTM_ERR_INVALID_ARG;
    const bool reverse = dir == LSTM_DIR_REVERSE;
    const int order = opt ? opt->gate_order : LSTM_GATES_IFJO;
    if (order != LSTM_GATES_IFJO && order != LSTM_GATES_IJFO) return LSTM_ERR_INVALID_ARG;
    const bool ijfo = order == LSTM_GATES_IJFO;
    if (!dims_supported(d)) return LSTM_ERR_UNSUPPORTED;
    const long long TB = (long long)d->T * d->B, BH = (long long)d->B * d->H;
    if (!ptr_ok(x, TB * d->I > 0) || !ptr_ok(W, d->H > 0) || !ptr_ok(b, false) ||
        !ptr_ok(h0, false) || !ptr_ok(c0, false) || !ptr_ok(mask, false) ||
        !ptr_ok(y, TB * d->H > 0) || !ptr_ok(hT, BH > 0) || !ptr_ok(cT, BH > 0) ||
        !ptr_ok(gates, TB * d->H > 0) || !ptr_ok(cells, TB * d->H > 0))
        return LSTM_ERR_INVALID_ARG;
    Rec2Plan plan3;
    const bool fused = fwd_fused_plan(d, mask != nullptr, plan3);
    const int wsrc = ws_ok(ws, ws_bytes, fused ? kCtrlBytes : fwd_layout(d).total);
    if (wsrc != LSTM_OK) return wsrc;
    cudaStream_t s = (cudaStream_t)stream;
    if (reset_barriers(ws, s) != cudaSuccess) return LSTM_ERR_CUDA;
    const Rec2Plan *p3 = fused ? &plan3 : nullptr;
    if (d->dtype == LSTM_F32)
        return fwd_simt<float>(d, (const float *)x, (const float *)W, (const float *)b,
                               (const float *)h0, c0, (const float *)mask, reverse, ijfo,
                               (float *)y, (float *)hT, cT, (float *)gates, cells, (char *)ws,
                               ws_bytes, p3, s);
    if (d->dtype == LSTM_F16) {
        typedef __half hf;
        return fwd_simt<hf>(d, (const hf *)x, (const hf *)W, (const hf *)b, (const hf *)h0, c0,
                            (const hf *)mask, reverse, ijfo, (hf *)y, (hf *)hT, cT, (hf *)gates,
                            cells, (char *)ws, ws_bytes, p3, s);
    }
    typedef __nv_bfloat16 bf;
    return fwd_simt<bf>(d, (const bf *)x, (const bf *)W, (const bf *)b, (const bf *)h0, c0,
                        (const bf *)mask, reverse, ijfo, (bf *)y, (bf *)hT, cT, (bf *)gates,
                        cells, (char *)ws, ws_bytes, p3, s);
}

int bwd_entry(const lstm_dims *d, const lstm_options *opt, const void *dy, const void *dhT,
              const float *dcT, const void *x, const void *W, const void *h0, const float *c0,
              const void *y, const void *gates, const float *cells, float *dx, float *dW,
              float *db, float *dh0, float *dc0, void *ws, size_t ws_bytes, void *stream) {
    if (!dims_ok(d)) return LSTM_ERR_INVALID_ARG;
    const void *mask = opt ? opt->seq_mask : nullptr;
    const int dir = opt ? opt->direction : LSTM_DIR_FORWARD;
    if (dir != LSTM_DIR_FORWARD && dir != LSTM_DIR_REVERSE) return LSTM_ERR_INVALID_ARG;
    const bool reverse = dir == LSTM_DIR_REVERSE;
    const int order = opt ? opt->gate_order : LSTM_GATES_IFJO;
    if (order != LSTM_GATES_IFJO && order != LSTM_GATES_IJFO) return LSTM_ERR_INVALID_ARG;
    const bool ijfo = order == LSTM_GATES_IJFO;
    if (!dims_supported(d)) return LSTM_ERR_UNSUPPORTED;
    const long long TB = (long long)d->T * d->B, BH = (long long)d->B * d->H;
    const long long G4 = 4LL * d->H, K = (long long)d->H + d->I;
    if (!ptr_ok(mask, false) || !ptr_ok(dy, false) || !ptr_ok(dhT, false) ||
        !ptr_ok(dcT, false) || !ptr_ok(x, TB * d->I > 0) || !ptr_ok(W, d->H > 0) ||
        !ptr_ok(h0, false) || !ptr_ok(c0, false) || !ptr_ok(y, TB * d->H > 0) ||
        !ptr_ok(gates, TB * d->H > 0) || !ptr_ok(cells, TB * d->H > 0) ||
        !ptr_ok(dx, TB * d->I > 0) || !ptr_ok(dW, G4 * K > 0) || !ptr_ok(db, G4 > 0) ||
        !ptr_ok(dh0, BH > 0) || !ptr_ok(dc0, BH > 0))
        return LSTM_ERR_INVALID_ARG;
    const int wsrc = ws_ok(ws, ws_bytes, bwd_layout(d).total);
    if (wsrc != LSTM_OK) return wsrc;
    cudaStream_t s = (cudaStream_t)stream;
    if (reset_barriers(ws, s) != cudaSuccess) return LSTM_ERR_CUDA;
    if (d->dtype == LSTM_F32)
        return bwd_simt<float>(d, (const float *)dy, (const float *)dhT, dcT, (const float *)x,
                               (const float *)W, (const float *)h0, c0, (const float *)mask,
                               reverse, ijfo, (const float *)y, (const float *)gates, cells, dx,
                               dW, db, dh0, dc0, (char *)ws, s);
    if (d->dtype == LSTM_F16) {
        typedef __half hf;
        return bwd_simt<hf>(d, (const hf *)dy, (const hf *)dhT, dcT, (const hf *)x,
                            (const hf *)W, (const hf *)h0, c0, (const hf *)mask, reverse, ijfo,
                            (const hf *)y, (const hf *)gates, cells, dx, dW, db, dh0, dc0,
                            (char *)ws, s);
    }
    typedef __nv_bfloat16 bf;
    return bwd_simt<bf>(d, (const bf *)dy, (const bf *)dhT, dcT, (const bf *)x, (const bf *)W,
                        (const bf *)h0, c0, (const bf *)mask, reverse, ijfo, (const bf *)y,
                        (const bf *)gates, cells, dx, dW, db, dh0, dc0, (char *)ws, s);
}
// ------------------------------------------------------- stacked layers
// Layer l of a stack: layer 0 has the caller's sizes, every later layer reads
// the H-wide outputs of the one below it.
lstm_dims layer_dims(const lstm_dims *d, int l) {
    lstm_dims e = *d;
    if (l > 0) e.I = d->H;
    return e;
}

// Per-layer slices of the [L][...] arrays start 16-byte aligned when B*H
// elements of every stored type are whole 16-byte groups.
bool stack_slices_aligned(const lstm_dims *d) {
    const long long BH = (long long)d->B * d->H;
    return (BH * (long long)esize(d)) % 16 == 0 && (BH * 4) % 16 == 0;
}

// Layer after layer: one layer's workspace, then the upper layer's dx (float)
// and its compute-type copy, the next lower layer's dy (seq_total bytes).
// Layer wavefront (16-bit stacks of 2 .. kMaxWave layers): the shared control
// block, one layer workspace per layer (their recurrences run at once), then
// per layer l >= 1 its dx (float) and the compute-type dy of layer l - 1
// (wave_total bytes).  total, the size query's answer, covers both; a smaller
// workspace of at least seq_total runs the layers one after another.
struct StackBwdLayout {
    size_t layer, dxbuf, dybuf, seq_total, wave_total, total;
    size_t xb, yb;  // one T*B*H float / compute-type buffer, 256-aligned
    size_t wave_region(int l) const { return kCtrlBytes + (size_t)l * layer; }
    size_t wave_dx(int l) const { return wave_bufs + (size_t)(l - 1) * (xb + yb); }
    size_t wave_dy(int l) const { return wave_dx(l + 1) + xb; }
    size_t wave_bufs = 0;
};
StackBwdLayout stack_bwd_layout(const lstm_dims *d, int L) {
    StackBwdLayout S;
    S.layer = align_up(bwd_layout(d).total, 256);
    if (L > 1) {
        const lstm_dims d1 = layer_dims(d, 1);
        S.layer = std::max(S.layer, align_up(bwd_layout(&d1).total, 256));
    }
    const size_t TBH = (size_t)d->T * d->B * d->H;
    S.xb = align_up(TBH * sizeof(float), 256);
    S.yb = align_up(TBH * esize(d), 256);
    S.dxbuf = S.dybuf = S.seq_total = S.layer;
    if (L > 1) {  // dx of the layer above (float) and its compute-type copy
        S.dybuf = S.dxbuf + S.xb;
        S.seq_total = S.dybuf + S.yb;
    }
    S.wave_total = 0;
    if (L > 1 && L <= kMaxWave && d->dtype != LSTM_F32) {
        S.wave_bufs = kCtrlBytes + (size_t)L * S.layer;
        S.wave_total = S.wave_bufs + (size_t)(L - 1) * (S.xb + S.yb);
    }
    S.total = std::max(S.seq_total, S.wave_total);
    return S;
}

size_t stack_fwd_ws(const lstm_dims *d, int L) {
    size_t n = fwd_layout(d).total;
    if (L > 1) {
        const lstm_dims d1 = layer_dims(d, 1);
        n = std::max(n, fwd_layout(&d1).total);
    }
    return n;
}

// Layer wavefront of the stacked forward.  Layer l's step t reads layer
// l-1's output at step t and its own state after step t-1, so layer l can run
// one block of steps behind layer l-1 instead of after all of it.  Each
// layer's recurrence is the fused forward kernel on a grid of at most half
// the SMs, launched once per chunk of consecutive steps on a stream of its
// own; chunk c of layer l is ordered after chunk c of layer l-1 by an event
// (no kernel waits on another kernel).  Each layer's plan takes at most half
// of the SMs and of the clusters that can be co-resident, so that two
// layers' launches run at once.  Both recurrences are latency bound,
// so two layers' chunks side by side each run at nearly their own speed.  A
// chunk continues its layer from the saved h and c of the step before it, and
// every launch has step counters of its own in the one control block.
// LSTM_ERR_UNSUPPORTED / LSTM_ERR_NOT_CORESIDENT: the caller runs the layers
// one after another instead (outputs are rewritten from scratch).
template <class E>
int stack_fwd_wave(const lstm_dims *d, int L, bool reverse, bool ijfo, const E *x,
                   const void *const *W, const void *const *b, const E *h0, const float *c0,
                   E *y, E *hT, float *cT, E *gates, float *cells, Ctrl *ctrl, cudaStream_t s) {
    if (L < 2 || env_is("LSTM_STACK_WAVE", '0')) return LSTM_ERR_UNSUPPORTED;
    const int T = d->T;
    const long long B = d->B, H = d->H, BH = B * H, TBH = (long long)T * BH;
    // layer 0 and the layers above it (whose input width is H)
    Rec2Plan P[2];
    for (int k = 0; k < 2; ++k) {
        const lstm_dims dk = layer_dims(d, k);
        if (!plan_fwd3(&dk, P[k], false, 2)) return LSTM_ERR_UNSUPPORTED;
    }
    auto counters = [&](int l) { return P[l > 0].G * P[l > 0].split; };
    int per_chunk = 0;  // step counters of one chunk of every layer
    for (int l = 0; l < L; ++l) per_chunk += counters(l);
    // chunks of at least 8 steps, at most kMaxWaveChunks, and every launch's
    // counters within the control block; LSTM_STACK_CHUNKS overrides (1: each
    // layer in one launch, the layers still ordered by events)
    const int nbar = (int)(sizeof(ctrl->bar) / sizeof(ctrl->bar[0]));
    const char *ov = getenv("LSTM_STACK_CHUNKS");
    int nch = ov ? atoi(ov) : std::min(kMaxWaveChunks, T / 8);
    nch = std::min(std::min(std::min(nch, kMaxWaveChunks), T), nbar / per_chunk);
    if (nch < (ov ? 1 : 2)) return LSTM_ERR_UNSUPPORTED;
    WaveStreams *Wv = wave_streams();
    if (!Wv) return LSTM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(Wv->mu);
    const int ns = std::min(L, kMaxWave);
    if (cudaEventRecord(Wv->fork, s) != cudaSuccess) return LSTM_ERR_CUDA;
    for (int l = 0; l < ns; ++l)
        if (cudaStreamWaitEvent(Wv->st[l], Wv->fork, 0) != cudaSuccess) return LSTM_ERR_CUDA;
    g_last_fwd_path = 3;
    g_last_stack_chunks = nch;
    int rc = LSTM_OK;
    for (int c = 0; c < nch && rc == LSTM_OK; ++c) {
        // steps [s0, s1): times [s0, s1), or [T - s1, T - s0) in reverse
        const int s0 = (int)((long long)c * T / nch), s1 = (int)((long long)(c + 1) * T / nch);
        const long long tlo = reverse ? T - s1 : s0;        // first time of the chunk
        const long long tprev = reverse ? T - s0 : s0 - 1;  // time of the step before it
        int bar = c * per_chunk;
        for (int l = 0; l < L && rc == LSTM_OK; ++l) {
            cudaStream_t sl = Wv->st[l % kMaxWave];
            if (l > 0 && cudaStreamWaitEvent(sl, Wv->ev[(l - 1) % kMaxWave][c], 0) != cudaSuccess) {
                rc = LSTM_ERR_CUDA;
                break;
            }
            lstm_dims dc = layer_dims(d, l);
            dc.T = s1 - s0;
            E *yl = y + l * TBH;
            float *cl = cells + l * TBH;
            const E *xc = l == 0 ? x + tlo * B * d->I : y + (l - 1) * TBH + tlo * BH;
            const E *h0c = c > 0 ? yl + tprev * BH : (h0 ? h0 + l * BH : nullptr);
            const float *c0c = c > 0 ? cl + tprev * BH : (c0 ? c0 + l * BH : nullptr);
            {
                prof::Phase ph(LSTM_PHASE_FWD_RECUR, sl);
                rc = tc_fwd_recurrence3(&dc, P[l > 0], xc, (const E *)W[l],
                                        b ? (const E *)b[l] : nullptr, h0c, c0c, (const E *)nullptr,
                                        reverse, ijfo, yl + tlo * BH, hT + l * BH, cT + l * BH,
                                        gates + 4 * (l * TBH + tlo * BH), cl + tlo * BH, ctrl, sl,
                                        bar);
            }
            bar += counters(l);
            if (rc == LSTM_OK && cudaEventRecord(Wv->ev[l % kMaxWave][c], sl) != cudaSuccess)
                rc = LSTM_ERR_CUDA;
        }
    }
    // join: nothing of this call stays unordered with the caller's stream
    for (int l = 0; l < ns; ++l)
        if (cudaEventRecord(Wv->join[l], Wv->st[l]) != cudaSuccess ||
            cudaStreamWaitEvent(s, Wv->join[l], 0) != cudaSuccess)
            return LSTM_ERR_CUDA;
    return rc;
}

// Layers 0 .. L-1 in order, each one lstm_fwd_ex call on the same stream.
int stack_fwd(const lstm_dims *d, int L, const lstm_options *opt, const void *x,
              const void *const *W, const void *const *b, const void *h0, const float *c0,
              void *y, void *hT, float *cT, void *gates, float *cells, void *ws, size_t ws_bytes,
              void *stream) {
    if (!dims_ok(d) || L < 1 || !W) return LSTM_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l)  // every layer's parameters, before any layer runs
        if (!ptr_ok(W[l], d->H > 0) || (b && !ptr_ok(b[l], false))) return LSTM_ERR_INVALID_ARG;
    if (L > 1 && !stack_slices_aligned(d)) return LSTM_ERR_UNSUPPORTED;
    const size_t es = esize(d);
    const long long BH = (long long)d->B * d->H, TBH = (long long)d->T * BH;
    g_last_stack_chunks = 0;
    // the layer wavefront where it applies (16-bit types, no length mask)
    const int dir = opt ? opt->direction : LSTM_DIR_FORWARD;
    const int order = opt ? opt->gate_order : LSTM_GATES_IFJO;
    if (L > 1 && d->dtype != LSTM_F32 && !(opt && opt->seq_mask) && dims_supported(d) &&
        (dir == LSTM_DIR_FORWARD || dir == LSTM_DIR_REVERSE) &&
        (order == LSTM_GATES_IFJO || order == LSTM_GATES_IJFO) && (long long)d->T * BH > 0 &&
        ptr_ok(x, (long long)d->T * d->B * d->I > 0) && ptr_ok(h0, false) && ptr_ok(c0, false) &&
        ptr_ok(y, true) && ptr_ok(hT, true) && ptr_ok(cT, true) && ptr_ok(gates, true) &&
        ptr_ok(cells, true) && ws_ok(ws, ws_bytes, kCtrlBytes) == LSTM_OK) {
        cudaStream_t s = (cudaStream_t)stream;
        if (reset_barriers(ws, s) != cudaSuccess) return LSTM_ERR_CUDA;
        const bool rev = dir == LSTM_DIR_REVERSE, ijfo = order == LSTM_GATES_IJFO;
        int rc;
        if (d->dtype == LSTM_F16)
            rc = stack_fwd_wave<__half>(d, L, rev, ijfo, (const __half *)x, W, b,
                                        (const __half *)h0, c0, (__half *)y, (__half *)hT, cT,
                                        (__half *)gates, cells, (Ctrl *)ws, s);
        else
            rc = stack_fwd_wave<bf16>(d, L, rev, ijfo, (const bf16 *)x, W, b, (const bf16 *)h0,
                                      c0, (bf16 *)y, (bf16 *)hT, cT, (bf16 *)gates, cells,
                                      (Ctrl *)ws, s);
        if (rc != LSTM_ERR_UNSUPPORTED && rc != LSTM_ERR_NOT_CORESIDENT) return rc;
        g_last_stack_chunks = 0;
    }
    const char *yb = static_cast<const char *>(y);
    for (int l = 0; l < L; ++l) {
        const lstm_dims dl = layer_dims(d, l);
        const void *xl = l == 0 ? x : yb + (size_t)(l - 1) * TBH * es;
        const int rc = fwd_entry(
            &dl, opt, xl, W[l], b ? b[l] : nullptr,
            h0 ? static_cast<const char *>(h0) + (size_t)l * BH * es : nullptr,
            c0 ? c0 + (size_t)l * BH : nullptr, static_cast<char *>(y) + (size_t)l * TBH * es,
            static_cast<char *>(hT) + (size_t)l * BH * es, cT + (size_t)l * BH,
            static_cast<char *>(gates) + (size_t)l * TBH * 4 * es, cells + (size_t)l * TBH, ws,
            ws_bytes, stream);
        if (rc != LSTM_OK) return rc;
    }
    return LSTM_OK;
}

// Layer wavefront of the stacked backward.  Layer l's reverse-time chunk c
// needs layer l+1's dx over the same times (its dy) and its own delta h,
// delta c after the chunk before, so it runs one chunk behind layer l+1
// instead of after all of it.  Per layer: the TMEM-weight backward recurrence
// on at most half the SMs and half the co-resident clusters (else two layers'
// launches would run one after the other), in the reverse-time chunks of the
// single-layer call, on a stream of its own; after each chunk, on a second stream, the dx
// GEMM over the chunk's rows and its rounding to the compute type into the
// lower layer's dy, which the lower layer's same chunk waits for (an event);
// on a third, low-priority stream the chunk's dW GEMM (with the stack's dx for
// layer 0).  No kernel waits on another kernel.  Every layer has its own
// workspace region and step counters in the one control block.
// LSTM_ERR_UNSUPPORTED / LSTM_ERR_NOT_CORESIDENT: the caller runs the layers
// one after another instead (every output is rewritten from scratch).
template <class E>
int stack_bwd_wave(const lstm_dims *d, int L, bool reverse, bool ijfo, const E *dy,
                   const E *dhT, const float *dcT, const E *x, const void *const *W, const E *h0,
                   const float *c0, const E *y, const E *gates, const float *cells, float *dx,
                   float *const *dW, float *const *db, float *dh0, float *dc0, char *ws,
                   size_t ws_bytes, cudaStream_t s) {
    if (L < 2 || L > kMaxWave || env_is("LSTM_STACK_WAVE", '0')) return LSTM_ERR_UNSUPPORTED;
    const StackBwdLayout S = stack_bwd_layout(d, L);
    if (S.wave_total == 0 || ws_bytes < S.wave_total) return LSTM_ERR_UNSUPPORTED;
    const int T = d->T, nsm = tcg::sm_count();
    const long long B = d->B, H = d->H, BH = B * H, TBH = (long long)T * BH, G4 = 4 * H;
    const int nch = bwd_chunks(d);
    if (nch < 2) return LSTM_ERR_UNSUPPORTED;
    Rec2Plan P[2];  // layer 0, the layers above it
    for (int k = 0; k < 2; ++k) {
        const lstm_dims dk = layer_dims(d, k);
        if (!tc_gemm_ok(&dk) ||
            !(plan_bwd4(&dk, P[k], 2) || plan_bwd3(&dk, P[k], 2)))
            return LSTM_ERR_UNSUPPORTED;
    }
    auto counters = [&](int l) { return P[l > 0].G * (P[l > 0].family == 4 ? 2 : 1); };
    auto rec_ctas = [&](int l) { return P[l > 0].R * P[l > 0].KS * P[l > 0].G; };
    int nbar = 0;
    for (int l = 0; l < L; ++l) nbar += counters(l);
    if (nbar > (int)(sizeof(((Ctrl *)nullptr)->bar) / sizeof(unsigned int)))
        return LSTM_ERR_UNSUPPORTED;
    WaveBwdStreams *Wv = wave_bwd_streams();
    if (!Wv) return LSTM_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(Wv->mu);
    Ctrl *ctrl = (Ctrl *)ws;
    if (reset_barriers(ws, s) != cudaSuccess) return LSTM_ERR_CUDA;
    // the GEMMs beside two layers' recurrences take at most the SMs those leave
    const int gemm_ctas = std::max(8, nsm - rec_ctas(0) - rec_ctas(std::min(1, L - 1)));
    if (cudaEventRecord(Wv->fork, s) != cudaSuccess) return LSTM_ERR_CUDA;
    for (int l = 0; l < L; ++l)
        if (cudaStreamWaitEvent(Wv->rec[l], Wv->fork, 0) != cudaSuccess ||
            cudaStreamWaitEvent(Wv->dxs[l], Wv->fork, 0) != cudaSuccess ||
            cudaStreamWaitEvent(Wv->gemm[l], Wv->fork, 0) != cudaSuccess)
            return LSTM_ERR_CUDA;
    g_last_bwd_path = P[L > 1].family;
    g_last_stack_bwd_chunks = nch;
    const BwdLayout Lb0 = bwd_layout(d);
    const lstm_dims d1 = layer_dims(d, 1);
    const BwdLayout Lb1 = bwd_layout(&d1);
    int rc = LSTM_OK;
    for (int c = 0; c < nch && rc == LSTM_OK; ++c) {
        const int i0 = chunk_bound(T, nch, c), i1 = chunk_bound(T, nch, c + 1);
        // times of the chunk's steps T-i1 .. T-i0-1 (i0 .. i1-1 in reverse)
        const long long t_lo = reverse ? i0 : T - i1, t_hi = reverse ? i1 : T - i0;
        int bar = nbar;
        for (int l = L - 1; l >= 0 && rc == LSTM_OK; --l) {
            bar -= counters(l);
            const lstm_dims dl = layer_dims(d, l);
            const BwdLayout &Lb = l == 0 ? Lb0 : Lb1;
            const Rec2Plan &Pl = P[l > 0];
            char *reg = ws + S.wave_region(l);
            E *dG = (E *)(reg + Lb.dG);
            E *WT = (E *)(reg + Lb.wt);
            float *dbgroup = (float *)(reg + Lb.dbgroup);
            const E *dyl = l == L - 1 ? dy : (const E *)(ws + S.wave_dy(l));
            const E *xl = l == 0 ? x : y + (l - 1) * TBH;
            const E *Wl = (const E *)W[l];
            const E *h0l = h0 ? h0 + l * BH : nullptr;
            const float *c0l = c0 ? c0 + l * BH : nullptr;
            cudaStream_t sr = Wv->rec[l], sx = Wv->dxs[l], sg = Wv->gemm[l];
            {
                prof::Phase ph(LSTM_PHASE_BWD_RECUR, sr);
                if (c == 0 && launch_transpose_wh(&dl, Wl, WT, sr) != cudaSuccess) {
                    rc = LSTM_ERR_CUDA;
                    break;
                }
                if (l < L - 1 && cudaStreamWaitEvent(sr, Wv->ev_dy[l][c], 0) != cudaSuccess) {
                    rc = LSTM_ERR_CUDA;
                    break;
                }
                rc = tc_bwd_tmem_launch(&dl, Pl, dyl, dhT ? dhT + l * BH : nullptr,
                                        dcT ? dcT + l * BH : nullptr, c0l, (const E *)nullptr,
                                        reverse, ijfo, gates + 4 * l * TBH, cells + l * TBH, dG, WT,
                                        dbgroup, dh0 + l * BH, dc0 + l * BH,
                                        (float *)(reg + Lb.dc), (float *)(reg + Lb.dhp), ctrl, i0,
                                        i1, sr, bar);
                if (rc != LSTM_OK) break;
                if (c + 1 == nch) {
                    simt::colsum_final<<<(unsigned)((G4 + 255) / 256), 256, 0, sr>>>(
                        dbgroup, Pl.G, (int)G4, db[l]);
                    note_launch();
                    if (cudaGetLastError() != cudaSuccess) rc = LSTM_ERR_CUDA;
                }
                if (rc == LSTM_OK && cudaEventRecord(Wv->ev_rec[l][c], sr) != cudaSuccess)
                    rc = LSTM_ERR_CUDA;
            }
            if (rc != LSTM_OK) break;
            if (l > 0) {  // this chunk's dx rows, rounded, are the lower layer's dy
                prof::Phase ph(LSTM_PHASE_DX, sx);
                float *dxl = (float *)(ws + S.wave_dx(l));
                E *dyb = (E *)(ws + S.wave_dy(l - 1));
                const long long n = (t_hi - t_lo) * BH;
                if (cudaStreamWaitEvent(sx, Wv->ev_rec[l][c], 0) != cudaSuccess ||
                    launch_hold(sx) != cudaSuccess ||
                    tc_dw_dx(&dl, (const E *)dG, xl, Wl, h0l, y + l * TBH, dW[l], dxl, ctrl, sx,
                             (int)t_lo, (int)t_hi, false, gemm_ctas, reverse, DX_PART) !=
                        cudaSuccess) {
                    rc = LSTM_ERR_CUDA;
                    break;
                }
                simt::from_float_copy<E><<<(unsigned)((n + 255) / 256), 256, 0, sx>>>(
                    dxl + t_lo * BH, dyb + t_lo * BH, n);
                note_launch();
                if (cudaGetLastError() != cudaSuccess ||
                    cudaEventRecord(Wv->ev_dy[l - 1][c], sx) != cudaSuccess) {
                    rc = LSTM_ERR_CUDA;
                    break;
                }
            }
            {   // the chunk's dW (accumulated from the second chunk on); layer 0 also dx
                prof::Phase ph(LSTM_PHASE_DW, sg);
                const bool alone = l == 0 && c + 1 == nch;  // nothing else left to run
                if (cudaStreamWaitEvent(sg, Wv->ev_rec[l][c], 0) != cudaSuccess ||
                    (!alone && launch_hold(sg) != cudaSuccess) ||
                    tc_dw_dx(&dl, (const E *)dG, xl, Wl, h0l, y + l * TBH, dW[l],
                             l == 0 ? dx : nullptr, ctrl, sg, (int)t_lo, (int)t_hi, c > 0,
                             alone ? 0 : gemm_ctas, reverse,
                             l == 0 ? (DW_PART | DX_PART) : DW_PART) != cudaSuccess)
                    rc = LSTM_ERR_CUDA;
            }
        }
    }
    // join: nothing of this call stays unordered with the caller's stream
    for (int l = 0; l < L; ++l) {
        cudaStream_t st[3] = {Wv->rec[l], Wv->dxs[l], Wv->gemm[l]};
        for (int k = 0; k < 3; ++k)
            if (cudaEventRecord(Wv->join[3 * l + k], st[k]) != cudaSuccess ||
                cudaStreamWaitEvent(s, Wv->join[3 * l + k], 0) != cudaSuccess)
                return LSTM_ERR_CUDA;
    }
    return rc;
}

// Layers L-1 .. 0, each one lstm_bwd_ex call; between two calls the float dx
// of the upper layer becomes the lower layer's dy in the compute type.
int stack_bwd(const lstm_dims *d, int L, const lstm_options *opt, const void *dy,
              const void *dhT, const float *dcT, const void *x, const void *const *W,
              const void *h0, const float *c0, const void *y, const void *gates,
              const float *cells, float *dx, float *const *dW, float *const *db, float *dh0,
              float *dc0, void *ws, size_t ws_bytes, void *stream) {
    if (!dims_ok(d) || L < 1 || !W || !dW || !db) return LSTM_ERR_INVALID_ARG;
    for (int l = 0; l < L; ++l) {  // every layer's parameters, before any layer runs
        const long long K = (long long)d->H + (l == 0 ? d->I : d->H);
        if (!ptr_ok(W[l], d->H > 0) || !ptr_ok(dW[l], 4LL * d->H * K > 0) ||
            !ptr_ok(db[l], d->H > 0))
            return LSTM_ERR_INVALID_ARG;
    }
    if (L > 1 && !stack_slices_aligned(d)) return LSTM_ERR_UNSUPPORTED;
    const StackBwdLayout S = stack_bwd_layout(d, L);
    const int wsrc = ws_ok(ws, ws_bytes, S.seq_total);
    if (wsrc != LSTM_OK) return wsrc;
    const size_t es = esize(d);
    const long long BH = (long long)d->B * d->H, TBH = (long long)d->T * BH;
    char *wsb = static_cast<char *>(ws);
    float *dxbuf = reinterpret_cast<float *>(wsb + S.dxbuf);
    void *dybuf = wsb + S.dybuf;
    cudaStream_t s = (cudaStream_t)stream;
    g_last_stack_bwd_chunks = 0;
    // the layer wavefront where it applies (16-bit types, no length mask, the
    // wavefront's workspace)
    const int dir = opt ? opt->direction : LSTM_DIR_FORWARD;
    const int order = opt ? opt->gate_order : LSTM_GATES_IFJO;
    if (L > 1 && d->dtype != LSTM_F32 && !(opt && opt->seq_mask) && dims_supported(d) &&
        (dir == LSTM_DIR_FORWARD || dir == LSTM_DIR_REVERSE) &&
        (order == LSTM_GATES_IFJO || order == LSTM_GATES_IJFO) && TBH > 0 &&
        ws_bytes >= S.wave_total && S.wave_total > 0 &&
        ptr_ok(dy, false) && ptr_ok(dhT, false) && ptr_ok(dcT, false) &&
        ptr_ok(x, (long long)d->T * d->B * d->I > 0) && ptr_ok(h0, false) && ptr_ok(c0, false) &&
        ptr_ok(y, true) && ptr_ok(gates, true) && ptr_ok(cells, true) &&
        ptr_ok(dx, (long long)d->T * d->B * d->I > 0) && ptr_ok(dh0, true) &&
        ptr_ok(dc0, true)) {
        const bool rev = dir == LSTM_DIR_REVERSE, ijfo = order == LSTM_GATES_IJFO;
        int rc;
        if (d->dtype == LSTM_F16)
            rc = stack_bwd_wave<__half>(d, L, rev, ijfo, (const __half *)dy, (const __half *)dhT,
                                        dcT, (const __half *)x, W, (const __half *)h0, c0,
                                        (const __half *)y, (const __half *)gates, cells, dx, dW,
                                        db, dh0, dc0, wsb, ws_bytes, s);
        else
            rc = stack_bwd_wave<bf16>(d, L, rev, ijfo, (const bf16 *)dy, (const bf16 *)dhT, dcT,
                                      (const bf16 *)x, W, (const bf16 *)h0, c0, (const bf16 *)y,
                                      (const bf16 *)gates, cells, dx, dW, db, dh0, dc0, wsb,
                                      ws_bytes, s);
        if (rc != LSTM_ERR_UNSUPPORTED && rc != LSTM_ERR_NOT_CORESIDENT) return rc;
        g_last_stack_bwd_chunks = 0;
    }
    for (int l = L - 1; l >= 0; --l) {
        const lstm_dims dl = layer_dims(d, l);
        const void *xl = l == 0 ? x : static_cast<const char *>(y) + (size_t)(l - 1) * TBH * es;
        const int rc = bwd_entry(
            &dl, opt, l == L - 1 ? dy : dybuf,
            dhT ? static_cast<const char *>(dhT) + (size_t)l * BH * es : nullptr,
            dcT ? dcT + (size_t)l * BH : nullptr, xl, W[l],
            h0 ? static_cast<const char *>(h0) + (size_t)l * BH * es : nullptr,
            c0 ? c0 + (size_t)l * BH : nullptr,
            static_cast<const char *>(y) + (size_t)l * TBH * es,
            static_cast<const char *>(gates) + (size_t)l * TBH * 4 * es, cells + (size_t)l * TBH,
            l == 0 ? dx : dxbuf, dW[l], db[l], dh0 + (size_t)l * BH, dc0 + (size_t)l * BH, ws,
            S.layer, stream);
        if (rc != LSTM_OK) return rc;
        if (l > 0 && TBH > 0) {
            const unsigned grid = (unsigned)((TBH + 255) / 256);
            if (d->dtype == LSTM_F32)
                simt::from_float_copy<float><<<grid, 256, 0, s>>>(dxbuf, (float *)dybuf, TBH);
            else if (d->dtype == LSTM_F16)
                simt::from_float_copy<__half><<<grid, 256, 0, s>>>(dxbuf, (__half *)dybuf, TBH);
            else
                simt::from_float_copy<bf16><<<grid, 256, 0, s>>>(dxbuf, (bf16 *)dybuf, TBH);
            note_launch();
            if (cudaGetLastError() != cudaSuccess) return LSTM_ERR_CUDA;
        }
    }
    return LSTM_OK;
}
}  // namespace

extern "C" {

int lstm_abi_version(void) { return LSTM_ABI_VERSION; }

const char *lstm_strerror(int code) {
    switch (code) {
        case LSTM_OK: return "ok";
        case LSTM_ERR_INVALID_ARG: return "invalid argument (dims, dtype, NULL or misaligned pointer)";
        case LSTM_ERR_UNSUPPORTED: return "unsupported configuration";
        case LSTM_ERR_WORKSPACE: return "workspace NULL, too small or not 256-byte aligned";
        case LSTM_ERR_CUDA: return "CUDA runtime error";
        case LSTM_ERR_TIMEOUT: return "device-side wait timed out";
        case LSTM_ERR_NOT_CORESIDENT: return "persistent grid cannot be co-resident";
        default: return "unknown status";
    }
}

size_t lstm_fwd_workspace_size(const lstm_dims *d) {
    if (!dims_ok(d)) return 0;
    return fwd_ws_need(d, false);
}

size_t lstm_fwd_workspace_size_ex(const lstm_dims *d, const lstm_options *opt) {
    if (!dims_ok(d)) return 0;
    return fwd_ws_need(d, opt && opt->seq_mask);
}

size_t lstm_fwd_workspace_size_max(const lstm_dims *d) {
    if (!dims_ok(d)) return 0;
    return fwd_layout(d).total;
}

size_t lstm_bwd_workspace_size(const lstm_dims *d) {
    if (!dims_ok(d)) return 0;
    return bwd_layout(d).total;
}


int lstm_fwd(const lstm_dims *d, const void *x, const void *W, const void *b, const void *h0,
             const float *c0, void *y, void *hT, float *cT, void *gates, float *cells, void *ws,
             size_t ws_bytes, void *stream) {
    return fwd_entry(d, nullptr, x, W, b, h0, c0, y, hT, cT, gates, cells, ws, ws_bytes, stream);
}

int lstm_fwd_ex(const lstm_dims *d, const lstm_options *opt, const void *x, const void *W,
                const void *b, const void *h0, const float *c0, void *y, void *hT, float *cT,
                void *gates, float *cells, void *ws, size_t ws_bytes, void *stream) {
    return fwd_entry(d, opt, x, W, b, h0, c0, y, hT, cT, gates, cells, ws, ws_bytes, stream);
}

int lstm_bwd(const lstm_dims *d, const void *dy, const void *dhT, const float *dcT,
             const void *x, const void *W, const void *h0, const float *c0, const void *y,
             const void *gates, const float *cells, float *dx, float *dW, float *db,
             float *dh0, float *dc0, void *ws, size_t ws_bytes, void *stream) {
    return bwd_entry(d, nullptr, dy, dhT, dcT, x, W, h0, c0, y, gates, cells, dx, dW, db, dh0,
                     dc0, ws, ws_bytes, stream);
}

int lstm_bwd_ex(const lstm_dims *d, const lstm_options *opt, const void *dy, const void *dhT,
                const float *dcT, const void *x, const void *W, const void *h0,
                const float *c0, const void *y, const void *gates, const float *cells,
                float *dx, float *dW, float *db, float *dh0, float *dc0, void *ws,
                size_t ws_bytes, void *stream) {
    return bwd_entry(d, opt, dy, dhT, dcT, x, W, h0, c0, y, gates, cells, dx, dW, db, dh0, dc0,
                     ws, ws_bytes, stream);
}

size_t lstm_stack_fwd_workspace_size(const lstm_dims *d, int L) {
    if (!dims_ok(d) || L < 1) return 0;
    return stack_fwd_ws(d, L);
}

size_t lstm_stack_bwd_workspace_size(const lstm_dims *d, int L) {
    if (!dims_ok(d) || L < 1) return 0;
    return stack_bwd_layout(d, L).total;
}

size_t lstm_stack_bwd_workspace_size_min(const lstm_dims *d, int L) {
    if (!dims_ok(d) || L < 1) return 0;
    return stack_bwd_layout(d, L).seq_total;
}

int lstm_stack_fwd(const lstm_dims *d, int L, const lstm_options *opt, const void *x,
                   const void *const *W, const void *const *b, const void *h0, const float *c0,
                   void *y, void *hT, float *cT, void *gates, float *cells, void *ws,
                   size_t ws_bytes, void *stream) {
    return stack_fwd(d, L, opt, x, W, b, h0, c0, y, hT, cT, gates, cells, ws, ws_bytes, stream);
}

int lstm_stack_bwd(const lstm_dims *d, int L, const lstm_options *opt, const void *dy,
                   const void *dhT, const float *dcT, const void *x, const void *const *W,
                   const void *h0, const float *c0, const void *y, const void *gates,
                   const float *cells, float *dx, float *const *dW, float *const *db,
                   float *dh0, float *dc0, void *ws, size_t ws_bytes, void *stream) {
    return stack_bwd(d, L, opt, dy, dhT, dcT, x, W, h0, c0, y, gates, cells, dx, dW, db, dh0,
                     dc0, ws, ws_bytes, stream);
}

int lstm_profile_begin(void) {
    for (auto &r : prof::g_recs) {
        prof::g_pool.push_back(r.a);
        prof::g_pool.push_back(r.b);
    }
    prof::g_recs.clear();
    prof::g_on = true;
    return LSTM_OK;
}

int lstm_profile_end(double *ms, long long *launches) {
    prof::g_on = false;
    if (ms)
        for (int i = 0; i < LSTM_NUM_PHASES; ++i) ms[i] = 0.0;
    if (launches)
        for (int i = 0; i < LSTM_NUM_PHASES; ++i) launches[i] = 0;
    int rc = LSTM_OK;
    for (auto &r : prof::g_recs) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) != cudaSuccess ||
            cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
            rc = LSTM_ERR_CUDA;
        if (ms) ms[r.phase] += t;
        if (launches) launches[r.phase] += r.launches;
        prof::g_pool.push_back(r.a);
        prof::g_pool.push_back(r.b);
    }
    prof::g_recs.clear();
    return rc;
}

long long lstm_launch_count(void) { return launch_counter().load(); }

int lstm_fwd_noalloc(const lstm_dims *d, const void *x, const void *W, const void *b,
                     const void *h0, const float *c0, void *y, void *hT, float *cT,
                     void *gates, float *cells, void *stream) {
    if (!dims_ok(d)) return LSTM_ERR_INVALID_ARG;
    if (!dims_supported(d)) return LSTM_ERR_UNSUPPORTED;
    if (fwd_ws_need(d, false) > (size_t)LSTM_NOALLOC_SCRATCH_BYTES) return LSTM_ERR_UNSUPPORTED;
    void *ws = nullptr;
    const int rc = noalloc_scratch(&ws);
    if (rc != LSTM_OK) return rc;
    // lstm_fwd checks every argument before it enqueues anything, then zeroes
    // the scratch's control block (status word, barrier counters) in stream
    // order: the previous call's bytes are never read
    return lstm_fwd(d, x, W, b, h0, c0, y, hT, cT, gates, cells, ws,
                    (size_t)LSTM_NOALLOC_SCRATCH_BYTES, stream);
}

int lstm_fwd_noalloc_status(void *stream) {
    void *ws = nullptr;
    const int rc = noalloc_scratch(&ws);
    if (rc != LSTM_OK) return rc;
    return lstm_status(ws, kCtrlBytes, stream);
}

int lstm_test_tc_gemm(int M, int N, int K, const void *A, long long lda, int a_mn_major,
                      const void *Bm, long long ldb, int b_mn_major, const void *bias, float *C,
                      long long ldc, void *ws, size_t ws_bytes, void *stream) {
    if (M < 0 || N < 0 || K < 0 || !A || !Bm || !C || !aligned16(A) || !aligned16(Bm) ||
        !ptr_ok(bias, false) || (lda % 8) || (ldb % 8))
        return LSTM_ERR_INVALID_ARG;
    if (!ws || ws_bytes < kCtrlBytes) return LSTM_ERR_WORKSPACE;
    if (!tcg::encode_fn()) return LSTM_ERR_UNSUPPORTED;
    tcg::Builder bld((Ctrl *)ws);
    // A: K-major = [M][K] (lda), MN-major = [K][M] (lda); B likewise with N.
    const int ma = a_mn_major ? bld.add_map({(const bf16 *)A, K, M, lda}, 1, 0)
                              : bld.add_map({(const bf16 *)A, M, K, lda}, 0, tcg::BM);
    const int mb = b_mn_major ? bld.add_map({(const bf16 *)Bm, K, N, ldb}, 1, 0)
                              : bld.add_map({(const bf16 *)Bm, N, K, ldb}, 0, tcg::BN);
    tcg::Problem &q = bld.add_problem(M, N, a_mn_major, b_mn_major, C, ldc, 0, (const bf16 *)bias);
    tcg::Builder::add_seg(q, ma, 0, mb, 0, K);
    if (!bld.ok) return LSTM_ERR_UNSUPPORTED;
    return tcg::launch(bld, (cudaStream_t)stream) == cudaSuccess ? LSTM_OK : LSTM_ERR_CUDA;
}

int lstm_test_set_wait_fault(int skip_cta, long long wait_ns) {
    g_fault_skip_cta = skip_cta;
    g_wait_ns = wait_ns > 0 ? (unsigned long long)wait_ns : 2000000000ull;
    return LSTM_OK;
}

int lstm_test_bwd_chunks(int T) {
    lstm_dims d = {T, 1, 1, 1, LSTM_BF16};
    return T < 0 ? -1 : bwd_chunks(&d);
}

int lstm_test_chunk_bound(int T, int nch, int c) {
    if (T < 0 || nch < 1 || c < 0 || c > nch) return -1;
    return chunk_bound(T, nch, c);
}

int lstm_test_last_stack_chunks(int *fwd_chunks, int *bwd_chunks) {
    if (fwd_chunks) *fwd_chunks = g_last_stack_chunks;
    if (bwd_chunks) *bwd_chunks = g_last_stack_bwd_chunks;
    return LSTM_OK;
}

int lstm_test_last_persist_split(int *fwd_ks, int *bwd_ks) {
    if (fwd_ks) *fwd_ks = g_last_pst_ks[0];
    if (bwd_ks) *bwd_ks = g_last_pst_ks[1];
    return LSTM_OK;
}

int lstm_test_last_paths(int *fwd_path, int *bwd_path) {
    if (fwd_path) *fwd_path = g_last_fwd_path;
    if (bwd_path) *bwd_path = g_last_bwd_path;
    return LSTM_OK;
}

int lstm_status(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < kCtrlBytes || ((uintptr_t)ws & 255u) != 0) return LSTM_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return LSTM_ERR_CUDA;
    unsigned int st = 0;
    if (cudaMemcpy(&st, ws, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return LSTM_ERR_CUDA;
    if (st != 0 && cudaMemset(ws, 0, 2 * sizeof(unsigned int)) != cudaSuccess) return LSTM_ERR_CUDA;
    return (int)st;
}

}  // extern "C"
