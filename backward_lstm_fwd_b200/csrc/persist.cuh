// persist.cuh -- persistent CUDA-core recurrences: all T steps of the forward
// recurrence, or of the backward recurrence, in one cooperative launch.
//
// They serve the compute types and shapes the tensor-core kernels do not:
// the fp32 compute type (the page's FLOAT; its 1e-4 tolerance rules out TF32
// products) and 16-bit shapes off the tensor-core grids.  Each step is the
// per-step kernel's work -- the contraction with W_h and the fused epilogue of
// simt.cuh (EpFwdStep: the forward-formula table; EpBwdStep: backward steps 1,
// 2, 3 and 5) -- so the epilogue arithmetic is shared, element for element.
// What differs is the schedule: the CTA that owns a slice of hidden units
// keeps that slice of W_h in shared memory (converted to fp32 once) for the
// whole call, every step streams the step's operand (h_{t-1} or dG_{t+1}, all
// batch rows, K in chunks) from L2, and the CTAs meet at a grid-wide
// step counter instead of a kernel boundary.  The per-step kernels put a
// B x 4H (or B x H) output on a few 64 x 64 tiles -- 4 CTAs for the backward
// step at B = 32, H = 256 -- and pay a launch per step; here every SM holds a
// slice of the units.
#pragma once

#include <type_traits>

#include "simt.cuh"
#include "tc_recur.cuh"  // rec::ld_acquire_u32 / red_release_add / wait_counter

namespace lstm {
namespace pst {

constexpr int NTHR = 256;
constexpr int MAXP = 4;         // (row, unit) pairs / (row, unit quad) items per thread
constexpr int STAGE_UNR = 8;    // operand loads in flight per thread while staging

// The step's operand is staged in K chunks of KC (a multiple of 32 the host
// picks so that a chunk of all B rows holds at most 16384 floats, within the
// shared memory left beside the weights), rows padded to KC + 1 floats so that
// rows m, m+1, ... start in different banks.  Each
// output item's dot product is split over KSPLIT lanes of one warp (a power of
// two <= 32 the host picks so that items x KSPLIT fill the CTA): lane `ks`
// of the group takes k = ks, ks + KSPLIT, ... of every chunk and the group's
// partial sums meet in a butterfly of shuffles.
// Forward: CTA c owns hidden units [c*UN, c*UN + UN) (all four gates).
// Shared memory: Ws [4][UN][H] fp32 (W_h rows g*H + j), hs [B][KC + 1] fp32.
__host__ __device__ inline size_t fwd_smem(int B, int H, int UN, int KC) {
    return (size_t)4 * UN * H * 4 + (size_t)B * (KC + 1) * 4;
}
// Backward: CTA c owns units [c*UN, c*UN + UN), UN a multiple of 4.
// Shared memory: Wt [UN][4H] fp32 (column j of W_h, all 4H rows), gs [B][KC + 1].
__host__ __device__ inline size_t bwd_smem(int B, int H, int UN, int KC) {
    return (size_t)UN * 4 * H * 4 + (size_t)B * (KC + 1) * 4;
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
    int T, B, H, I, UN, KC, KSPLIT, reverse, fb;
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
    Ctrl *ctrl;
    int T, B, H, I, UN, KC, KSPLIT, reverse, fb;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// Grid-wide step barrier: this CTA's arrival for `step` (release, after a
// CTA barrier that orders every thread's stores before it), and the wait for
// all CTAs' arrivals for `step` (acquire).  Bounded; false on time-out.
__device__ __forceinline__ bool grid_step(unsigned int *ctr, unsigned int target, bool arrive,
                                          Ctrl *ctrl, volatile int *abort_flag, uint32_t site,
                                          unsigned long long wait_ns) {
    __syncthreads();
    __shared__ int ok_s;
    if (threadIdx.x == 0) {
        if (arrive) rec::red_release_add(ctr, 1u);
        ok_s = rec::wait_counter(ctr, target, ctrl, abort_flag, site, wait_ns);
    }
    __syncthreads();
    return ok_s != 0;
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
// `ld` into dst[B][KC + 1] as fp32 (zeros past kn), by all threads, with
// STAGE_UNR independent loads in flight per thread: 16-byte loads when every
// row's slice starts on a 16-byte boundary and holds whole vectors, else
// element loads.
template <class T>
__device__ __forceinline__ void stage_chunk(float *dst, const T *src, long long ld, int B, int k0,
                                            int kn, int KC) {
    const int KCP = KC + 1;
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
                    for (int i = 0; i < V; ++i) dst[m * KCP + kk + i] = f[i];
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

template <class T>
__global__ void __launch_bounds__(NTHR, 1) fwd_kernel(const FwdParams<T> p) {
    extern __shared__ float4 smem_f4[];
    float *Ws = reinterpret_cast<float *>(smem_f4);
    const int H = p.H, B = p.B, T_ = p.T, UN = p.UN, KC = p.KC, KCP = KC + 1;
    const int KSPLIT = p.KSPLIT, slot = threadIdx.x / KSPLIT, ks = threadIdx.x % KSPLIT;
    const int nslots = NTHR / KSPLIT;
    float *hs = Ws + (size_t)4 * UN * H;
    __shared__ int abort_s;
    if (threadIdx.x == 0) abort_s = 0;
    const int j0 = blockIdx.x * UN;
    const int un = min(UN, H - j0);  // units this CTA owns (the last CTA may own fewer)
    const long long K = (long long)H + p.I;
    // W_h rows g*H + j0 + jj, all H columns, converted to fp32
    for (int e = threadIdx.x; e < 4 * UN * H; e += NTHR) {
        const int k = e % H, r = e / H, jj = r % UN, g = r / UN;
        Ws[e] = jj < un ? to_f(p.W[((long long)g * H + j0 + jj) * K + k]) : 0.f;
    }
    unsigned int *ctr = &p.ctrl->bar[0];
    const unsigned int P = gridDim.x;
    const int npairs = B * un;  // pair q -> row m = q % B, unit jj = q / B
    auto tau = [&](int st) { return p.reverse ? T_ - 1 - st : st; };
    const long long BH = (long long)B * H;
    for (int st = 0; st < T_; ++st) {
        const int t = tau(st), tp = p.reverse ? t + 1 : t - 1;
        const T *hp = st > 0 ? p.y + (long long)tp * BH : p.h0;
        float acc[MAXP][4];
#pragma unroll
        for (int i = 0; i < MAXP; ++i)
#pragma unroll
            for (int g = 0; g < 4; ++g) acc[i][g] = 0.f;
        if (hp) {
            for (int k0 = 0; k0 < H; k0 += KC) {
                const int kn = min(KC, H - k0);
                __syncthreads();  // the previous chunk has been read
                stage_chunk(hs, hp, H, B, k0, kn, KC);
                __syncthreads();
#pragma unroll
                for (int i = 0; i < MAXP; ++i) {
                    const int q = slot + i * nslots;
                    if (q >= npairs) break;
                    const int m = q % B, jj = q / B;
                    const float *hrow = hs + m * KCP;
                    const float *w0 = Ws + ((size_t)0 * UN + jj) * H + k0;
                    const float *w1 = Ws + ((size_t)1 * UN + jj) * H + k0;
                    const float *w2 = Ws + ((size_t)2 * UN + jj) * H + k0;
                    const float *w3 = Ws + ((size_t)3 * UN + jj) * H + k0;
                    for (int kk = ks; kk < kn; kk += KSPLIT) {
                        const float h = hrow[kk];
                        acc[i][0] = fmaf(h, w0[kk], acc[i][0]);
                        acc[i][1] = fmaf(h, w1[kk], acc[i][1]);
                        acc[i][2] = fmaf(h, w2[kk], acc[i][2]);
                        acc[i][3] = fmaf(h, w3[kk], acc[i][3]);
                    }
                }
            }
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
        group_sum(acc, KSPLIT);
#pragma unroll
        for (int i = 0; i < MAXP; ++i) {
            const int q = slot + i * nslots;
            if (q >= npairs) break;
            const int m = q % B, jj = q / B;
            if (ks == 0) ep(m, 4 * (j0 + jj), acc[i]);
        }
        // h_t of every unit is the next step's operand: grid barrier
        if (st + 1 < T_) {
            const bool arrive = (int)blockIdx.x != p.fault_skip_cta;
            if (!grid_step(ctr, P * (unsigned)(st + 1), arrive, p.ctrl, &abort_s, 0xA01, p.wait_ns))
                return;
        }
    }
}

template <class T>
__global__ void __launch_bounds__(NTHR, 1) bwd_kernel(const BwdParams<T> p) {
    extern __shared__ float4 smem_f4[];
    float *Wt = reinterpret_cast<float *>(smem_f4);
    const int H = p.H, B = p.B, T_ = p.T, UN = p.UN, KC = p.KC, KCP = KC + 1;
    const int KSPLIT = p.KSPLIT, slot = threadIdx.x / KSPLIT, ks = threadIdx.x % KSPLIT;
    const int nslots = NTHR / KSPLIT;
    const int G4 = 4 * H;
    float *gs = Wt + (size_t)UN * G4;
    __shared__ int abort_s;
    if (threadIdx.x == 0) abort_s = 0;
    const int j0 = blockIdx.x * UN;
    const long long K = (long long)H + p.I;
    // column j0 + jj of W_h, all 4H rows, converted to fp32 (zero past H)
    for (int e = threadIdx.x; e < UN * G4; e += NTHR) {
        const int k = e % G4, jj = e / G4;
        Wt[e] = j0 + jj < H ? to_f(p.W[(long long)k * K + j0 + jj]) : 0.f;
    }
    unsigned int *ctr = &p.ctrl->bar[0];
    const unsigned int P = gridDim.x;
    const int nq = UN / 4;          // unit quads of this CTA
    const int nitems = B * nq;      // item q -> row m = q % B, quad jq = q / B
    auto tau = [&](int st) { return p.reverse ? T_ - 1 - (long long)st : (long long)st; };
    const long long BH = (long long)B * H;
    for (int st = T_ - 1; st >= 0; --st) {
        const bool last = st == T_ - 1;
        const long long t = tau(st);
        float acc[MAXP][4];
#pragma unroll
        for (int i = 0; i < MAXP; ++i)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;
        if (!last) {
            // delta h = dG_{t_next} W_h for this CTA's units
            const T *dGn = p.dG + tau(st + 1) * B * G4;
            for (int k0 = 0; k0 < G4; k0 += KC) {
                const int kn = min(KC, G4 - k0);
                __syncthreads();
                stage_chunk(gs, dGn, G4, B, k0, kn, KC);
                __syncthreads();
#pragma unroll
                for (int i = 0; i < MAXP; ++i) {
                    const int q = slot + i * nslots;
                    if (q >= nitems) break;
                    const int m = q % B, jq = q / B;
                    const float *grow = gs + m * KCP;
                    const float *w0 = Wt + (size_t)(4 * jq + 0) * G4 + k0;
                    const float *w1 = Wt + (size_t)(4 * jq + 1) * G4 + k0;
                    const float *w2 = Wt + (size_t)(4 * jq + 2) * G4 + k0;
                    const float *w3 = Wt + (size_t)(4 * jq + 3) * G4 + k0;
                    for (int kk = ks; kk < kn; kk += KSPLIT) {
                        const float g = grow[kk];
                        acc[i][0] = fmaf(g, w0[kk], acc[i][0]);
                        acc[i][1] = fmaf(g, w1[kk], acc[i][1]);
                        acc[i][2] = fmaf(g, w2[kk], acc[i][2]);
                        acc[i][3] = fmaf(g, w3[kk], acc[i][3]);
                    }
                }
            }
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
        group_sum(acc, KSPLIT);
#pragma unroll
        for (int i = 0; i < MAXP; ++i) {
            const int q = slot + i * nslots;
            if (q >= nitems) break;
            const int m = q % B, jq = q / B;
            if (ks == 0) ep(m, j0 + 4 * jq, acc[i]);
        }
        // dG_t of every unit is the next step's operand: grid barrier
        if (st > 0) {
            const bool arrive = (int)blockIdx.x != p.fault_skip_cta;
            if (!grid_step(ctr, P * (unsigned)(T_ - st), arrive, p.ctrl, &abort_s, 0xA02,
                           p.wait_ns))
                return;
        }
    }
}

}  // namespace pst
}  // namespace lstm
