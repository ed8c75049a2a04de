// persist.cuh -- persistent CUDA-core recurrences: all T steps of the forward
// recurrence, or of the backward recurrence, in one cooperative launch.
//
// They serve the compute types and shapes the tensor-core kernels do not:
// the fp32 compute type (the page's FLOAT; its 1e-4 tolerance rules out TF32
// products) and 16-bit shapes off the tensor-core grids.  Each step is the
// per-step kernel's work -- the contraction with W_h and the fused epilogue of
// simt.cuh (EpFwdStep: the forward-formula table; EpBwdStep: backward steps 1,
// 2, 3 and 5) -- so the epilogue arithmetic is shared, element for element.
// What differs is the schedule.  A cluster of KS CTAs owns UC = KS * UN hidden
// units and splits the contraction's K axis (H for h_{t-1} W_h^T, 4H for
// dG_{t+1} W_h) into KS slices: CTA r keeps slice r of the cluster's weights
// in shared memory (converted to fp32 once) for the whole call, and every step
// streams only slice r of the step's operand (all batch rows) from L2.  Its
// partial sums for the units CTA o finishes go to o by one bulk DSMEM copy
// (slot r of o's receive block, one mbarrier with expected bytes), each CTA
// adds the KS slots of its own UN units in rank order and runs the epilogue,
// and all CTAs meet at a grid-wide step counter.  With KS = 1 there is no
// exchange: the CTA streams the whole operand.  The per-step kernels instead
// put a B x 4H (or B x H) output on a few 64 x 64 tiles and pay a launch per
// step.
#pragma once

#include <type_traits>

#include "simt.cuh"
#include "tc_recur.cuh"  // rec::ld_acquire_u32 / red_release_add / wait_counter

namespace lstm {
namespace pst {

constexpr int NTHR = 256;
constexpr int MAXP = 8;         // contraction items per thread
constexpr int STAGE_UNR = 8;    // operand loads in flight per thread while staging

// Work split of one launch (host and device).
//   KS      CTAs per cluster, each taking one K slice (1: no split)
//   UN      units whose epilogue a CTA runs (a multiple of 4 in the backward,
//           whose epilogue works on quads of units)
//   KSL     K-slice length, a multiple of 8 (the last slice may hold fewer
//           real columns; weights past K are zero)
//   KC      staging chunk: columns of the slice staged at once for all B rows,
//           a multiple of 32
//   KCP     row pitch of the staged chunk in floats: KC + 4 * min(KSPLIT, 8),
//           so that the rows a quarter warp reads start in different banks
//   KSPLIT  lanes of a warp that share one item's dot product (a power of two;
//           lane ks takes float4 columns ks, ks + KSPLIT, ...), their partial
//           sums meeting in a butterfly of shuffles
// Contraction items: forward (row m, unit u of the cluster) with the four gate
// rows of u; backward (row m, quad of units) with one dot product per unit.
struct Split {
    int KS, UN, KSL, KC, KCP, KSPLIT;
};

// Floats of one CTA's partial block for one owner: forward B x UN x 4 gates,
// backward B x UN units.
__host__ __device__ inline int part_floats(bool bwd, int B, int UN) {
    return bwd ? B * UN : 4 * B * UN;
}

// Shared-memory plan in floats from the (16-byte aligned) dynamic base:
// weights, staged operand chunk, KS - 1 send blocks, KS receive slots, the
// receive mbarrier.  Every region starts on a 16-byte boundary.
struct Layout {
    int w, opnd, stage, recv, bar;
    size_t bytes;
};
__host__ __device__ inline Layout layout(bool bwd, int B, const Split &s) {
    const int UC = s.KS * s.UN;
    const int part = part_floats(bwd, B, s.UN);
    Layout L;
    L.w = 0;
    L.opnd = (bwd ? 1 : 4) * UC * s.KSL;
    L.stage = L.opnd + B * s.KCP;
    L.recv = L.stage + (s.KS - 1) * part;
    L.bar = L.recv + s.KS * part;
    L.bytes = (size_t)(L.bar + 4) * 4;
    return L;
}

template <class E>
struct FwdParams {
    const E *W;            // [4H][H + I]
    const float *Gx;       // [T*B][4H] (input projection with the bias)
    const E *h0;           // [B][H] or NULL
    const float *c0;       // [B][H] or NULL
    const E *mask;         // [T][B][H] or NULL
    E *y, *gates;
    float *cells;
    Ctrl *ctrl;
    int T, B, H, I, reverse, fb;
    Split s;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

template <class E>
struct BwdParams {
    const E *W;            // [4H][H + I]
    const E *dy, *dhT, *gates, *mask;
    const float *dcT, *cells, *c0;
    E *dG;                 // [T*B][4H]
    float *dcbuf[2];       // delta c ping-pong [B][H]
    float *dc0;            // [B][H]: delta c after the first step (dinitC)
    float *dhpbuf[2];      // delta h passed on by padding, ping-pong [B][H]
    float *dh0;            // [B][H]: dinitH = W_h^T dG of the first step (+ padding's share)
    Ctrl *ctrl;
    int T, B, H, I, reverse, fb;
    Split s;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// Grid-wide step barrier: this CTA's arrival for `step` (release, after a
// CTA barrier that orders every thread's stores before it), then `meanwhile`
// by every thread (work that must not delay the arrival), then the wait for
// all CTAs' arrivals for `step` (acquire).  Bounded; false on time-out.
template <class Fn>
__device__ __forceinline__ bool grid_step(unsigned int *ctr, unsigned int target, bool arrive,
                                          Ctrl *ctrl, volatile int *abort_flag, uint32_t site,
                                          unsigned long long wait_ns, Fn meanwhile) {
    __syncthreads();
    __shared__ int ok_s;
    if (threadIdx.x == 0 && arrive) rec::red_release_add(ctr, 1u);
    meanwhile();
    if (threadIdx.x == 0) ok_s = rec::wait_counter(ctr, target, ctrl, abort_flag, site, wait_ns);
    __syncthreads();
    return ok_s != 0;
}

// Partial sums to their owners: every thread calls this after the writers
// have put this CTA's partials for itself in receive slot r and those for the
// other CTAs in the send blocks (send block sp goes to rank r + 1 + sp, so
// that each CTA receives from one sender at a time).  Thread 0 posts the
// expected bytes and issues the copies; every thread waits (bounded) for the
// other ranks' copies into this CTA, and thread 0 for its own copies to have
// read their sources, so the send blocks may be refilled afterwards.
__device__ __forceinline__ bool exchange(float *stage, float *recv, uint64_t *bar, uint32_t &rph,
                                         int KS, int r, int part_bytes, Ctrl *ctrl,
                                         volatile int *abort_flag, uint32_t site,
                                         unsigned long long wait_ns) {
    if (KS == 1) {
        __syncthreads();
        return true;
    }
    tc::fence_proxy_async_smem();  // these generic stores, then the copies' async reads
    __syncthreads();
    if (threadIdx.x == 0) {
        tc::mbar_arrive_expect_tx(bar, (uint32_t)((KS - 1) * part_bytes));
        const uint32_t recv_lo = tc::smem_u32(recv), bar_lo = tc::smem_u32(bar);
        for (int sp = 0; sp < KS - 1; ++sp) {
            const uint32_t d = (uint32_t)((r + 1 + sp) % KS);
            tc::bulk_copy_to_peer(tc::map_rank(recv_lo + (uint32_t)(r * part_bytes), d),
                                  stage + sp * (part_bytes / 4), (uint32_t)part_bytes,
                                  tc::map_rank(bar_lo, d));
        }
        tc::bulk_commit();
    }
    const bool ok = tc::mbar_wait_cluster(bar, rph, ctrl, abort_flag, site, wait_ns);
    rph ^= 1;
    if (threadIdx.x == 0) tc::bulk_wait_read_all();
    return __syncthreads_and(ok) != 0;
}

// 16 bytes of T as floats: the element type of one vector load
__device__ __forceinline__ void to_f4(const float4 &v, float *o) {
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
template <class T>
__device__ __forceinline__ void to_f8(const uint4 &v, float *o) {
    const T *e = reinterpret_cast<const T *>(&v);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = to_f(e[i]);
}

// Rows [0, B) x columns [k0, k0 + kn) of a row-major operand with row pitch
// `ld` into dst[B][KCP] as fp32 (zeros in columns kn .. KC - 1), by all
// threads, with STAGE_UNR independent loads in flight per thread: 16-byte
// loads when every row's slice starts on a 16-byte boundary and holds whole
// vectors, else element loads.
template <class T>
__device__ __forceinline__ void stage_chunk(float *dst, const T *src, long long ld, int B, int k0,
                                            int kn, int KC, int KCP) {
    constexpr int V = 16 / (int)sizeof(T);  // elements per 16-byte load
    if (KC % V == 0 && kn % V == 0 && k0 % V == 0 && ld % V == 0 &&
        ((uintptr_t)src & 15u) == 0) {
        const int vpr = KC / V, nv = B * vpr;  // vectors per row, per chunk
        for (int base = threadIdx.x; base < nv; base += NTHR * STAGE_UNR) {
            typedef typename std::conditional<sizeof(T) == 4, float4, uint4>::type Vt;
            Vt v[STAGE_UNR];
#pragma unroll
            for (int u = 0; u < STAGE_UNR; ++u) {
                const int e = base + u * NTHR;
                const int m = e / vpr, kk = (e - m * vpr) * V;
                if (e < nv && kk < kn)
                    v[u] = *reinterpret_cast<const Vt *>(src + (long long)m * ld + k0 + kk);
                else
                    memset(&v[u], 0, sizeof(Vt));
            }
#pragma unroll
            for (int u = 0; u < STAGE_UNR; ++u) {
                const int e = base + u * NTHR;
                if (e < nv) {
                    const int m = e / vpr, kk = (e - m * vpr) * V;
                    float f[V];
                    if constexpr (sizeof(T) == 4) to_f4(v[u], f);
                    else to_f8<T>(v[u], f);
#pragma unroll
                    for (int i = 0; i < V; i += 4)
                        *reinterpret_cast<float4 *>(dst + m * KCP + kk + i) =
                            make_float4(f[i], f[i + 1], f[i + 2], f[i + 3]);
                }
            }
        }
        return;
    }
    const int n = B * KC;
    for (int base = threadIdx.x; base < n; base += NTHR * STAGE_UNR) {
        float v[STAGE_UNR];
#pragma unroll
        for (int u = 0; u < STAGE_UNR; ++u) {
            const int e = base + u * NTHR;
            const int m = e / KC, kk = e - m * KC;
            v[u] = (e < n && kk < kn) ? to_f(src[(long long)m * ld + k0 + kk]) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < STAGE_UNR; ++u) {
            const int e = base + u * NTHR;
            if (e < n) {
                const int m = e / KC;
                dst[m * KCP + (e - m * KC)] = v[u];
            }
        }
    }
}

// Sum of the four accumulators of each item over the KSPLIT lanes of its
// group (every lane of the warp takes part; each ends with the group's sums).
__device__ __forceinline__ void group_sum(float (&acc)[MAXP][4], int ksplit) {
    for (int off = ksplit / 2; off > 0; off /= 2)
#pragma unroll
        for (int i = 0; i < MAXP; ++i)
#pragma unroll
            for (int g = 0; g < 4; ++g)
                acc[i][g] += __shfl_xor_sync(0xffffffffu, acc[i][g], off);
}

// Pull one line of read-only input into this SM's L1 ahead of its use.
__device__ __forceinline__ void prefetch_l1(const void *ptr) {
    asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr));
}

__device__ __forceinline__ float dot4(const float4 &a, const float4 &b, float acc) {
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    return fmaf(a.w, b.w, acc);
}

// acc[i][c] += sum over the chunk of opnd row m(i) times weight row wrow(i, c):
// items q = slot + i * nslots < nitems; lane ks of the item's group takes the
// float4 columns ks, ks + KSPLIT, ... < nv (columns past the chunk are zero in
// both operands).
template <class RowFn>
__device__ __forceinline__ void contract(float (&acc)[MAXP][4], const float *opnd, int KCP,
                                         int nitems, int B, int slot, int nslots, int ks,
                                         int KSPLIT, int nv, RowFn wrow) {
#pragma unroll
    for (int i = 0; i < MAXP; ++i) {
        const int q = slot + i * nslots;
        if (q >= nitems) break;
        const int m = q % B, it = q / B;
        const float4 *o4 = reinterpret_cast<const float4 *>(opnd + m * KCP);
        const float4 *w0 = reinterpret_cast<const float4 *>(wrow(it, 0));
        const float4 *w1 = reinterpret_cast<const float4 *>(wrow(it, 1));
        const float4 *w2 = reinterpret_cast<const float4 *>(wrow(it, 2));
        const float4 *w3 = reinterpret_cast<const float4 *>(wrow(it, 3));
        for (int v = ks; v < nv; v += KSPLIT) {
            const float4 h = o4[v];
            acc[i][0] = dot4(h, w0[v], acc[i][0]);
            acc[i][1] = dot4(h, w1[v], acc[i][1]);
            acc[i][2] = dot4(h, w2[v], acc[i][2]);
            acc[i][3] = dot4(h, w3[v], acc[i][3]);
        }
    }
}

// Shared prologue of both kernels: the CTA's abort flag and, with KS > 1, the
// receive mbarrier, initialised before any peer may complete bytes on it.
__device__ __forceinline__ void init_exchange(uint64_t *rbar, int KS, volatile int *abort_s) {
    if (threadIdx.x == 0) {
        *abort_s = 0;
        if (KS > 1) {
            tc::mbar_init(rbar, 1);
            tc::fence_mbar_init();
        }
    }
}

// Last act of both kernels, on every path: no copy of this CTA in flight, and
// with KS > 1 no CTA of the cluster leaves while a peer may still copy into it.
__device__ __forceinline__ void finish_exchange(int KS) {
    if (KS > 1 && threadIdx.x == 0) tc::bulk_wait_all();
    __syncthreads();
    if (KS > 1) tc::cluster_sync_all();
}

template <class T>
__global__ void __launch_bounds__(NTHR, 1) fwd_kernel(const FwdParams<T> p) {
    extern __shared__ float4 smem_f4[];
    float *sm = reinterpret_cast<float *>(smem_f4);
    const Split &sp = p.s;
    const int H = p.H, B = p.B, T_ = p.T, KS = sp.KS, UN = sp.UN, UC = KS * UN;
    const int KSL = sp.KSL, KC = sp.KC, KCP = sp.KCP, KSPLIT = sp.KSPLIT;
    const int slot = threadIdx.x / KSPLIT, ks = threadIdx.x % KSPLIT, nslots = NTHR / KSPLIT;
    const Layout L = layout(false, B, sp);
    float *Ws = sm + L.w, *hs = sm + L.opnd, *stage = sm + L.stage, *recv = sm + L.recv;
    uint64_t *rbar = reinterpret_cast<uint64_t *>(sm + L.bar);
    __shared__ int abort_s;
    const int r = KS > 1 ? (int)tc::cluster_rank() : 0;
    const int u0 = (int)(blockIdx.x / KS) * UC;    // first unit of the cluster
    const int k_lo = r * KSL, kl = min(KSL, H - k_lo);  // this CTA's columns of h (<= 0: none)
    const long long K = (long long)H + p.I;
    init_exchange(rbar, KS, &abort_s);
    // Ws[g][u][kk] = W_h[g*H + u0 + u][k_lo + kk] in fp32, zero past H
    for (int e = threadIdx.x; e < 4 * UC * KSL; e += NTHR) {
        const int kk = e % KSL, row = e / KSL, u = row % UC, g = row / UC;
        Ws[e] = (u0 + u < H && kk < kl)
                    ? to_f(p.W[((long long)g * H + u0 + u) * K + k_lo + kk]) : 0.f;
    }
    if (KS > 1) tc::cluster_sync_all();
    else __syncthreads();
    unsigned int *ctr = &p.ctrl->bar[0];
    const unsigned int P = gridDim.x;
    const int nitems = B * UC, part = part_floats(false, B, UN);
    auto tau = [&](int st) { return p.reverse ? T_ - 1 - st : st; };
    auto wrow = [&](int u, int g) { return Ws + (size_t)(g * UC + u) * KSL; };
    const long long BH = (long long)B * H;
    uint32_t rph = 0;
    for (int st = 0; st < T_; ++st) {
        const int t = tau(st), tp = p.reverse ? t + 1 : t - 1;
        const T *hp = st > 0 ? p.y + (long long)tp * BH : p.h0;
        const bool contracted = hp != nullptr;  // h_{-1} = 0 otherwise: no product
        if (contracted) {
            float acc[MAXP][4];
#pragma unroll
            for (int i = 0; i < MAXP; ++i)
#pragma unroll
                for (int g = 0; g < 4; ++g) acc[i][g] = 0.f;
            for (int c0 = 0; c0 < kl; c0 += KC) {
                const int kn = min(KC, kl - c0);
                __syncthreads();  // the previous chunk has been read
                stage_chunk(hs, hp, H, B, k_lo + c0, kn, KC, KCP);
                __syncthreads();
                contract(acc, hs, KCP, nitems, B, slot, nslots, ks, KSPLIT, (kn + 3) >> 2,
                         [&](int u, int g) { return wrow(u, g) + c0; });
            }
            group_sum(acc, KSPLIT);
            if (ks == 0) {
#pragma unroll
                for (int i = 0; i < MAXP; ++i) {
                    const int q = slot + i * nslots;
                    if (q >= nitems) break;
                    const int m = q % B, u = q / B, o = u / UN, ul = u - o * UN;
                    float *dst = o == r ? recv + r * part : stage + ((o - r - 1 + KS) % KS) * part;
                    *reinterpret_cast<float4 *>(dst + (m * UN + ul) * 4) =
                        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
                }
            }
            if (!exchange(stage, recv, rbar, rph, KS, r, part * 4, p.ctrl, &abort_s, 0xA03,
                          p.wait_ns))
                break;
        }
        simt::EpFwdStep<T> ep{p.Gx + (long long)t * B * 4 * H,
                              st > 0 ? p.cells + (long long)tp * BH : p.c0,
                              p.y + (long long)t * BH, p.gates + (long long)t * B * 4 * H,
                              p.cells + (long long)t * BH, H};
        if (p.mask) {
            ep.mask = p.mask + (long long)t * BH;
            ep.hprev = hp;
        }
        ep.fb = p.fb;
        // the epilogue of this CTA's own units: the KS slots summed in rank order
        for (int e = threadIdx.x; e < B * UN; e += NTHR) {
            const int m = e % B, ul = e / B;
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            if (contracted)
                for (int sl = 0; sl < KS; ++sl) {
                    const float4 v = *reinterpret_cast<const float4 *>(recv + sl * part +
                                                                       (m * UN + ul) * 4);
                    a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
                }
            ep(m, 4 * (u0 + r * UN + ul), a);
        }
        // h_t of every unit is the next step's operand: grid barrier; after
        // this CTA's arrival, the next step's read-only epilogue inputs of its
        // units (Gx, mask) go into L1 while it waits
        if (st + 1 < T_) {
            const bool arrive = (int)blockIdx.x != p.fault_skip_cta;
            const long long tn = tau(st + 1);
            auto prefetch = [&]() {
                for (int e = threadIdx.x; e < B * UN; e += NTHR) {
                    const int m = e % B, j = u0 + r * UN + e / B;
                    if (j >= H) continue;
                    const float *gx = p.Gx + (tn * B + m) * 4 * H + j;
#pragma unroll
                    for (int g = 0; g < 4; ++g) prefetch_l1(gx + g * H);
                    if (p.mask) prefetch_l1(p.mask + tn * BH + (long long)m * H + j);
                }
            };
            if (!grid_step(ctr, P * (unsigned)(st + 1), arrive, p.ctrl, &abort_s, 0xA01, p.wait_ns,
                           prefetch))
                break;
        }
    }
    finish_exchange(KS);
}

template <class T>
__global__ void __launch_bounds__(NTHR, 1) bwd_kernel(const BwdParams<T> p) {
    extern __shared__ float4 smem_f4[];
    float *sm = reinterpret_cast<float *>(smem_f4);
    const Split &sp = p.s;
    const int H = p.H, B = p.B, T_ = p.T, KS = sp.KS, UN = sp.UN, UC = KS * UN;
    const int KSL = sp.KSL, KC = sp.KC, KCP = sp.KCP, KSPLIT = sp.KSPLIT;
    const int slot = threadIdx.x / KSPLIT, ks = threadIdx.x % KSPLIT, nslots = NTHR / KSPLIT;
    const int G4 = 4 * H, QN = UN / 4;  // quads of units a CTA finishes
    const Layout L = layout(true, B, sp);
    float *Wt = sm + L.w, *gs = sm + L.opnd, *stage = sm + L.stage, *recv = sm + L.recv;
    uint64_t *rbar = reinterpret_cast<uint64_t *>(sm + L.bar);
    __shared__ int abort_s;
    const int r = KS > 1 ? (int)tc::cluster_rank() : 0;
    const int u0 = (int)(blockIdx.x / KS) * UC;     // first unit of the cluster
    const int k_lo = r * KSL, kl = min(KSL, G4 - k_lo);  // this CTA's columns of dG
    const long long K = (long long)H + p.I;
    init_exchange(rbar, KS, &abort_s);
    // Wt[u][kk] = W_h[k_lo + kk][u0 + u] (column u0 + u of W_h) in fp32, zero past 4H / H
    for (int e = threadIdx.x; e < UC * KSL; e += NTHR) {
        const int kk = e % KSL, u = e / KSL;
        Wt[e] = (u0 + u < H && kk < kl) ? to_f(p.W[(long long)(k_lo + kk) * K + u0 + u]) : 0.f;
    }
    if (KS > 1) tc::cluster_sync_all();
    else __syncthreads();
    unsigned int *ctr = &p.ctrl->bar[0];
    const unsigned int P = gridDim.x;
    const int nitems = B * (UC / 4), part = part_floats(true, B, UN);
    auto tau = [&](int st) { return p.reverse ? T_ - 1 - (long long)st : (long long)st; };
    const long long BH = (long long)B * H;
    uint32_t rph = 0;
    // steps T-1 .. 0, then st = -1: dinitH = W_h^T dG of step 0, the same
    // contraction and exchange with only a store after it
    for (int st = T_ - 1; st >= -1; --st) {
        const bool last = st == T_ - 1;  // no dG_{t+1}: delta h comes from dhT
        const long long t = st >= 0 ? tau(st) : 0;
        if (!last) {
            // delta h = dG_{t_next} W_h, this CTA's K slice, for the cluster's units
            float acc[MAXP][4];
#pragma unroll
            for (int i = 0; i < MAXP; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
            const T *dGn = p.dG + tau(st + 1) * B * G4;
            for (int c0 = 0; c0 < kl; c0 += KC) {
                const int kn = min(KC, kl - c0);
                __syncthreads();
                stage_chunk(gs, dGn, G4, B, k_lo + c0, kn, KC, KCP);
                __syncthreads();
                contract(acc, gs, KCP, nitems, B, slot, nslots, ks, KSPLIT, (kn + 3) >> 2,
                         [&](int jq, int c) { return Wt + (size_t)(4 * jq + c) * KSL + c0; });
            }
            group_sum(acc, KSPLIT);
            if (ks == 0) {
#pragma unroll
                for (int i = 0; i < MAXP; ++i) {
                    const int q = slot + i * nslots;
                    if (q >= nitems) break;
                    const int m = q % B, jq = q / B, o = jq / QN, lq = jq - o * QN;
                    float *dst = o == r ? recv + r * part : stage + ((o - r - 1 + KS) % KS) * part;
                    *reinterpret_cast<float4 *>(dst + (m * QN + lq) * 4) =
                        make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
                }
            }
            if (!exchange(stage, recv, rbar, rph, KS, r, part * 4, p.ctrl, &abort_s, 0xA04,
                          p.wait_ns))
                break;
        }
        if (st < 0) {
            for (int e = threadIdx.x; e < B * QN; e += NTHR) {
                const int m = e % B, lq = e / B;
                const float4 v0 = *reinterpret_cast<const float4 *>(recv + (m * QN + lq) * 4);
                float a[4] = {v0.x, v0.y, v0.z, v0.w};
                for (int sl = 1; sl < KS; ++sl) {
                    const float4 v = *reinterpret_cast<const float4 *>(recv + sl * part +
                                                                       (m * QN + lq) * 4);
                    a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
                }
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int j = u0 + r * UN + 4 * lq + c;
                    if (j >= H) continue;
                    const long long o = (long long)m * H + j;
                    p.dh0[o] = a[c] + (p.mask ? p.dhpbuf[0][o] : 0.f);
                }
            }
            break;
        }
        simt::EpBwdStep<T> ep;
        ep.dy = p.dy ? p.dy + t * BH : nullptr;
        ep.dh_in = last ? p.dhT : nullptr;
        ep.dc_in = last ? p.dcT : p.dcbuf[(st + 1) & 1];
        ep.gates = p.gates + t * B * G4;
        ep.cells = p.cells + t * BH;
        ep.cprev = st > 0 ? p.cells + tau(st - 1) * BH : p.c0;
        ep.dG = p.dG + t * B * G4;
        ep.dc_out = st == 0 ? p.dc0 : p.dcbuf[st & 1];
        ep.H = H;
        ep.use_acc = !last;
        ep.fb = p.fb;
        if (p.mask) {
            ep.mask = p.mask + t * BH;
            ep.dhp_in = last ? nullptr : p.dhpbuf[(st + 1) & 1];
            ep.dhp_out = p.dhpbuf[st & 1];
        }
        // the epilogue of this CTA's own quads: the KS slots summed in rank order
        for (int e = threadIdx.x; e < B * QN; e += NTHR) {
            const int m = e % B, lq = e / B;
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            if (!last)
                for (int sl = 0; sl < KS; ++sl) {
                    const float4 v = *reinterpret_cast<const float4 *>(recv + sl * part +
                                                                       (m * QN + lq) * 4);
                    a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
                }
            ep(m, u0 + r * UN + 4 * lq, a);
        }
        // dG_t of every unit is the next step's operand: grid barrier; after
        // this CTA's arrival, the next step's read-only epilogue inputs of its
        // units (gates, cells, c_{t-1}, dy, mask) go into L1 while it waits
        {
            const bool arrive = (int)blockIdx.x != p.fault_skip_cta;
            const long long tn = st > 0 ? tau(st - 1) : 0;
            auto prefetch = [&]() {
                for (int e = threadIdx.x; st > 0 && e < B * QN; e += NTHR) {
                    const int m = e % B, j = u0 + r * UN + 4 * (e / B);
                    if (j >= H) continue;
                    const long long o = (long long)m * H + j;
                    const T *g4 = p.gates + (tn * B + m) * G4 + j;
#pragma unroll
                    for (int g = 0; g < 4; ++g) prefetch_l1(g4 + g * H);
                    prefetch_l1(p.cells + tn * BH + o);
                    if (st - 1 > 0) prefetch_l1(p.cells + tau(st - 2) * BH + o);
                    else if (p.c0) prefetch_l1(p.c0 + o);
                    if (p.dy) prefetch_l1(p.dy + tn * BH + o);
                    if (p.mask) prefetch_l1(p.mask + tn * BH + o);
                }
            };
            if (!grid_step(ctr, P * (unsigned)(T_ - st), arrive, p.ctrl, &abort_s, 0xA02,
                           p.wait_ns, prefetch))
                break;
        }
    }
    finish_exchange(KS);
}

}  // namespace pst
}  // namespace lstm
