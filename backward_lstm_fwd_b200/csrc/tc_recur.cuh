// tc_recur.cuh -- persistent tcgen05 kernel of the forward recurrence (bf16):
// for t = 0..T-1,  pre = Gx_t + h_{t-1} W_h^T,  i,f,o = sigma, g = tanh,
// c_t = f c_{t-1} + i g,  h_t = o tanh(c_t)   ("SingleLayerLstmGrad",
// forward-formula table).
//
// Decomposition: CTA (s, gi) owns hidden units j0 = 16 s .. j0 + 15 for all
// four gates -- 64 rows of W_h, kept resident in shared memory for all T steps
// (A operand, K-major, 128-byte swizzle) -- and the batch rows
// b0 = gi * NB .. b0 + NB - 1.  Per step the 64 x NB gate block is one chain of
// tcgen05.mma (M = 64, N = NB, K = 16) over H, with h_{t-1} = y[t-1] streamed by
// TMA through a ring of 64-wide K chunks.  The CTAs of one batch group hand
// h_t to each other through global memory (L2) and one counter: each CTA adds 1
// (release) after storing its part of y[t]; the next step's loads wait for
// S * (t+1) arrivals (acquire, bounded).  Groups never wait on each other.
//
// Warp roles (192 threads):
//   warp 0     producer: W_h slice once, then per step wait for the group,
//              stream h_{t-1};
//   warp 1     TMEM owner; one thread issues the MMAs into one of two
//              accumulators (alternating per step);
//   warps 2-5  epilogue: TMEM -> gate exchange in smem -> + Gx_t, activations,
//              cell and hidden update, stores of y, gates, cells (c stays in
//              registers across steps), then the group arrival.
//
// TMEM layout of an M = 64 accumulator: row m sits in lane 32 * (m / 16) + m % 16,
// column n in column n.  Rows are ordered m = 16 * gate + unit, so the warp with
// lane quarter q reads gate q of the 16 units in its lanes 0..15.
#pragma once

#include "tc_ptx.cuh"

namespace lstm {
namespace rec {

constexpr int UNITS = 16;              // hidden units per CTA
constexpr int MROWS = 4 * UNITS;       // 64: the MMA's M
constexpr int KCH_BYTES = MROWS * 128; // one 64-wide K chunk of the W slice: 8 KB
constexpr int NUM_THREADS = 192;
constexpr int EPI_THREADS = 128;

struct FwdParams {
    CUtensorMap map_w;    // W [4H][H+I], box {64, 16}
    CUtensorMap map_y;    // y [T*B][H], box {64, NB}
    CUtensorMap map_h0;   // h0 [B][H], box {64, NB} (valid only if has_h0)
    const float *Gx;      // [T*B][4H]
    const float *c0;      // [B][H] or NULL
    __nv_bfloat16 *y, *gates, *hT;
    float *cells, *cT;
    Ctrl *ctrl;
    int T, B, H, S, G, kch, stages, has_h0;
    int fault_skip_cta;   // test hook: this CTA never arrives (-1: none)
    unsigned long long wait_ns;
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int *p) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void red_release_add(unsigned int *p, unsigned int v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void named_bar(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// AND of `v` over the N epilogue threads (named barrier 2), so that every
// epilogue thread takes the same branch after a bounded wait.
template <int N>
__device__ __forceinline__ bool epi_vote_all_n(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "n"(N)
        : "memory");
    return r != 0;
}

// AND of `v` over the 128 epilogue threads (named barrier 2), so that every
// epilogue thread takes the same branch after a bounded wait -- no thread is
// left alone at a later barrier or warp-synchronous TMEM load.
__device__ __forceinline__ bool epi_vote_all(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 2, 128, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v)
        : "memory");
    return r != 0;
}

// Activations of the bf16 recurrent kernels: the hardware tanh approximation
// (MUFU, about 2^-11 relative error, well below bf16's 2^-8 storage step) and
// the logistic function through the identity sigma(x) = (1 + tanh(x / 2)) / 2.
__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float sigmoid_fast(float x) { return fmaf(0.5f, tanh_fast(0.5f * x), 0.5f); }

// Wait until *ctr >= target (acquire).  Bounded by limit_ns of %globaltimer;
// on time-out record LSTM_ERR_TIMEOUT with `site` and raise the abort flag.
__device__ __forceinline__ bool wait_counter(const unsigned int *ctr, unsigned int target,
                                             Ctrl *ctrl, volatile int *abort_flag,
                                             uint32_t site, unsigned long long limit_ns) {
    if (ld_acquire_u32(ctr) >= target) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    while (true) {
        // 32 polls per look at the clock and the abort flag: reading
        // %globaltimer on every poll made the step barrier's detection slower
        // (the recurrences 1.8 % slower per step on the bench workload)
        for (int k = 0; k < 32; ++k)
            if (ld_acquire_u32(ctr) >= target) return true;
        if (*abort_flag) return false;
        if (tc::globaltimer_ns() - t0 > limit_ns) {
            atomicCAS(&ctrl->status, 0u, 5u);
            atomicCAS(&ctrl->fail_site, 0u, site);
            *abort_flag = 1;
            return false;
        }
    }
}

// Shared-memory plan (bytes from the 1024-aligned base).
// The gate-exchange buffer (4 x NB x 16 fp32) aliases the ring: the ring is
// idle between the last MMA of a step and the group barrier of the next one,
// which is exactly when the epilogue uses the buffer.
constexpr int MAX_STAGES = 16;
constexpr int BAR_BYTES = 512;
struct FwdSmem {
    int w, ring, xbuf, bars, total;
    __host__ __device__ FwdSmem(int kch, int stages, int NB) {
        w = 0;
        ring = kch * KCH_BYTES;
        xbuf = ring;
        const int ring_bytes = stages * NB * 128, x_bytes = 4 * NB * UNITS * 4;
        bars = ring + (ring_bytes > x_bytes ? ring_bytes : x_bytes);
        total = bars + BAR_BYTES;
    }
};

template <int NB>
__global__ void __launch_bounds__(NUM_THREADS, 1) fwd_kernel(const __grid_constant__ FwdParams p) {
    constexpr int NK = NB / 8;  // (unit, batch) pairs per epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const FwdSmem L(p.kch, p.stages, NB);
    uint8_t *sW = smem + L.w;
    uint8_t *ring = smem + L.ring;
    float *xbuf = (float *)(smem + L.xbuf);
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *full = bars;                  // [stages]
    uint64_t *empty = bars + MAX_STAGES;    // [stages]
    uint64_t *w_full = bars + 2 * MAX_STAGES;
    uint64_t *mma_done = w_full + 1;        // [2]
    uint32_t *tmem_slot = (uint32_t *)(mma_done + 3);
    volatile int *abort_flag = (volatile int *)(mma_done + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int s = blockIdx.x % p.S, gi = blockIdx.x / p.S;
    const int j0 = s * UNITS, b0 = gi * NB;
    const int H = p.H, B = p.B;
    unsigned int *ctr = &p.ctrl->bar[gi];
    constexpr uint32_t TMEM_COLS = (2 * NB < 32) ? 32 : 2 * NB;
    // every CTA of a group walks the K chunks from a different start, so that
    // concurrent TMA requests spread over the L2 slices
    const int rot = (s * 5 + gi * 3) % p.kch;

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(w_full, 1);
        tc::mbar_init(&mma_done[0], 1);
        tc::mbar_init(&mma_done[1], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---- the resident W_h slice: rows g*H + j0 .. +15, all H columns
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(p.kch * KCH_BYTES));
            for (int kc = 0; kc < p.kch; ++kc)
                for (int g = 0; g < 4; ++g)
                    tc::tma_load_2d(sW + kc * KCH_BYTES + g * UNITS * 128, &p.map_w, w_full,
                                    64 * kc, g * H + j0);
            // ---- per step: h_{t-1} chunks into the ring
            uint32_t stage = 0, phase = 0;
            bool aborted = false;
            for (int t = 0; t < p.T; ++t) {
                if (t > 0) {
                    if (!wait_counter(ctr, (unsigned)(p.S * t), p.ctrl, abort_flag, 0x201,
                                      p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    // the group's generic-proxy stores were released to this
                    // thread's acquire; order the TMA (async-proxy) reads after it
                    tc::fence_proxy_async_global();
                } else if (!p.has_h0) {
                    continue;  // h_{-1} = 0: no MMA at t = 0
                }
                const CUtensorMap *m = t > 0 ? &p.map_y : &p.map_h0;
                const int row0 = t > 0 ? (t - 1) * B + b0 : b0;
                bool ok = true;
                int kc = rot;
                for (int ic = 0; ic < p.kch; ++ic, kc = (kc + 1 == p.kch) ? 0 : kc + 1) {
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, p.ctrl, abort_flag, 0x202,
                                       p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[stage], NB * 128);
                    tc::tma_load_2d(ring + stage * NB * 128, m, &full[stage], 64 * kc, row0);
                    if (++stage == (uint32_t)p.stages) stage = 0, phase ^= 1;
                }
                if (!ok) {
                    aborted = true;
                    break;
                }
            }
            if (aborted) {
                // let the copies already issued land before the CTA can exit
                tc::mbar_wait(w_full, 0, nullptr, nullptr, 0, 200000000ull);
                for (int i = 0; i < p.stages; ++i) {
                    if (stage == 0) stage = p.stages, phase ^= 1;
                    --stage;
                    tc::mbar_wait(&full[stage], phase, nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // descriptors = base + integer offsets (see tc_gemm.cuh); the issuing
            // thread is on every step's critical path
            uint32_t stage = 0, phase = 0;
            const uint32_t idesc = tc::idesc_bf16_f32(MROWS, NB, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t w_lo0 = tc::smem_u32(sW) >> 4, r_lo0 = tc::smem_u32(ring) >> 4;
            constexpr uint32_t WSTEP = KCH_BYTES >> 4, RSTEP = (NB * 128) >> 4;
            bool ok = tc::mbar_wait(w_full, 0, p.ctrl, abort_flag, 0x203, p.wait_ns);
            for (int t = 0; ok && t < p.T; ++t) {
                const int acc = t & 1;
                if (t == 0 && !p.has_h0) {
                    tc::mbar_arrive(&mma_done[acc]);
                    continue;
                }
                const uint32_t d = tmem_base + acc * NB;
                int kc = rot;
                for (int ic = 0; ic < p.kch; ++ic, kc = (kc + 1 == p.kch) ? 0 : kc + 1) {
                    if (!tc::mbar_wait(&full[stage], phase, p.ctrl, abort_flag, 0x204, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t ad = hi | (w_lo0 + kc * WSTEP);
                    const uint64_t bd = hi | (r_lo0 + stage * RSTEP);
                    tc::mma_bf16(d, ad, bd, idesc, ic != 0);
                    tc::mma_bf16(d, ad + 2, bd + 2, idesc, 1);
                    tc::mma_bf16(d, ad + 4, bd + 4, idesc, 1);
                    tc::mma_bf16(d, ad + 6, bd + 6, idesc, 1);
                    tc::mma_commit(&empty[stage]);
                    if (++stage == (uint32_t)p.stages) stage = 0, phase ^= 1;
                }
                if (ok) tc::mma_commit(&mma_done[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;        // 0..127
        const int q = warp & 3;                 // TMEM lane quarter = gate of the rows read
        const int u = et % UNITS;               // unit of this thread's pairs
        const int nq = et / UNITS;              // pairs n = nq + 8 k
        const int j = j0 + u;
        float c[NK], gx[4][NK];
#pragma unroll
        for (int k = 0; k < NK; ++k) {
            const int b = b0 + nq + 8 * k;
            c[k] = (p.c0 && b < B) ? p.c0[(long long)b * H + j] : 0.f;
        }
        auto load_gx = [&](int t) {
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                const int b = b0 + nq + 8 * k;
                const float *row = p.Gx + ((long long)t * B + b) * 4 * H + j;
#pragma unroll
                for (int g = 0; g < 4; ++g) gx[g][k] = (b < B) ? __ldg(row + g * H) : 0.f;
            }
        };
        load_gx(0);
        for (int t = 0; t < p.T; ++t) {
            const int acc = t & 1;
            const bool w = tc::mbar_wait(&mma_done[acc], (t >> 1) & 1, p.ctrl, abort_flag, 0x205,
                                         p.wait_ns);
            if (!epi_vote_all(w)) break;
            tc::tc_fence_after();
            const bool zero = (t == 0 && !p.has_h0);
            // TMEM rows of this warp: gate q, unit = lane (lanes 0..15); all
            // loads in flight before one wait
            constexpr int CB = NB < 64 ? NB : (NB >= 128 ? 32 : 64);  // columns per wait
#pragma unroll
            for (int cb = 0; cb < NB; cb += CB) {
                uint32_t r[CB / 16][16];
#pragma unroll
                for (int c = 0; c < CB / 16; ++c)
                    tc::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + acc * NB + cb + 16 * c,
                                  r[c]);
                tc::tmem_ld_wait();
                if (lane < UNITS) {
#pragma unroll
                    for (int c = 0; c < CB / 16; ++c)
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            xbuf[(q * NB + cb + 16 * c + i) * UNITS + lane] =
                                zero ? 0.f : __uint_as_float(r[c][i]);
                }
            }
            tc::tc_fence_before();
            named_bar(1, EPI_THREADS);
            __nv_bfloat16 *yt = p.y + (long long)t * B * H;
            __nv_bfloat16 *gt = p.gates + (long long)t * B * 4 * H;
            float *ct = p.cells + (long long)t * B * H;
#pragma unroll
            for (int k = 0; k < NK; ++k) {
                const int n = nq + 8 * k, b = b0 + n;
                const float ig = sigmoid_fast(xbuf[(0 * NB + n) * UNITS + u] + gx[0][k]);
                const float fg = sigmoid_fast(xbuf[(1 * NB + n) * UNITS + u] + gx[1][k]);
                const float gg = tanh_fast(xbuf[(2 * NB + n) * UNITS + u] + gx[2][k]);
                const float og = sigmoid_fast(xbuf[(3 * NB + n) * UNITS + u] + gx[3][k]);
                c[k] = fg * c[k] + ig * gg;
                const float h = og * tanh_fast(c[k]);
                if (b < B) {
                    const long long o = (long long)b * H + j;
                    yt[o] = __float2bfloat16_rn(h);
                    ct[o] = c[k];
                    __nv_bfloat16 *g4 = gt + (long long)b * 4 * H + j;
                    g4[0] = __float2bfloat16_rn(ig);
                    g4[H] = __float2bfloat16_rn(fg);
                    g4[2 * H] = __float2bfloat16_rn(gg);
                    g4[3 * H] = __float2bfloat16_rn(og);
                    if (t == p.T - 1) {
                        p.hT[o] = __float2bfloat16_rn(h);
                        p.cT[o] = c[k];
                    }
                }
            }
            if (t + 1 < p.T) load_gx(t + 1);
            named_bar(1, EPI_THREADS);       // all of y[t] stored; xbuf free again
            if (et == 0 && (int)blockIdx.x != p.fault_skip_cta) {
                red_release_add(ctr, 1u);  // release: the step's stores, ordered by bar.sync
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}


// ===========================================================================
// Persistent tcgen05 kernel of the backward recurrence (bf16), "SingleLayerLstmGrad"
// backward algorithm steps 1-3, 5 and 6, with db (step 4) accumulated on the way:
// for t = T-1 .. 0
//   delta h_t  = dy_t + (t == T-1 ? dhT : dG_{t+1} W_h)          (steps 1, 5, 6)
//   delta c_t  = delta h_t o (1 - tanh^2 c_t) + delta c_next      (step 2)
//   do, dg, di, df                                                (step 3)
//   delta c_next = delta c_t f_t                                  (steps 5, 6)
// and finally dh0 = dG_0 W_h, dc0 = delta c_next.
//
// Decomposition: CTA (s, gi) owns hidden units j0 = 16 s .. j0 + 15 and batch
// rows b0 = gi * NB .. b0 + NB - 1 (NB <= 64).  Its product is
// D[64 batch rows, 16 units] = dG_{t+1}[rows, 0:4H] . W_h[0:4H, units]: A = the
// dG rows, TMA-streamed in 64-wide K chunks after the group barrier; B = the
// CTA's 16 rows of W_h^T (a transposed copy in the workspace), resident in
// shared memory (K-major, 128-byte swizzle).  Only the first NB rows of each A
// chunk are loaded; the rest of the 64-row tile is stale and its output rows
// are never read.  dG_t of all units is exchanged through global memory with
// one release/acquire counter per batch group, exactly as in the forward kernel.
//
// Epilogue thread (q, lane): batch row m = 16 q + lane % 16 (the TMEM lane of
// that row in an M = 64 accumulator), units j0 + 8 * (lane / 16) .. + 7; lanes
// 16..31 receive their eight values from lane - 16 by shuffle.
// ===========================================================================

constexpr int BWD_STAGE_BYTES = 64 * 128;  // one 64-row x 64-wide A chunk
constexpr int WT_CHUNK_BYTES = UNITS * 128;

struct BwdParams {
    CUtensorMap map_wt;   // W_h^T [H][4H], box {64, 16}
    CUtensorMap map_dg;   // dG [T*B][4H], box {64, NB}
    const __nv_bfloat16 *dy, *dhT, *gates;
    const float *dcT, *cells, *c0;
    __nv_bfloat16 *dG;
    float *dh0, *dc0, *db_part;  // db_part [G][4H]
    Ctrl *ctrl;
    int T, B, H, S, G, NB, kch4, stages;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

struct BwdSmem {
    int wt, ring, bars, total;
    __host__ __device__ BwdSmem(int kch4, int stages) {
        wt = 0;
        ring = kch4 * WT_CHUNK_BYTES;
        bars = ring + stages * BWD_STAGE_BYTES;
        total = bars + BAR_BYTES;
    }
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = __bfloat1622float2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
__device__ __forceinline__ uint4 f32x8_to_bf16(const float (&f)[8]) {
    uint4 v;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return v;
}

__global__ void __launch_bounds__(NUM_THREADS, 1) bwd_kernel(const __grid_constant__ BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const BwdSmem L(p.kch4, p.stages);
    uint8_t *sWT = smem + L.wt;
    uint8_t *ring = smem + L.ring;
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *full = bars;
    uint64_t *empty = bars + MAX_STAGES;
    uint64_t *w_full = bars + 2 * MAX_STAGES;
    uint64_t *mma_done = w_full + 1;
    uint32_t *tmem_slot = (uint32_t *)(mma_done + 3);
    volatile int *abort_flag = (volatile int *)(mma_done + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int s = blockIdx.x % p.S, gi = blockIdx.x / p.S;
    const int j0 = s * UNITS, b0 = gi * p.NB;
    const int H = p.H, B = p.B, T = p.T, NB = p.NB;
    unsigned int *ctr = &p.ctrl->bar[gi];
    constexpr uint32_t TMEM_COLS = 32;  // two 16-column accumulators
    const int rot = (s * 5 + gi * 3) % p.kch4;  // spread concurrent TMA requests over L2

    if (threadIdx.x == 0) {
        for (int i = 0; i < p.stages; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(w_full, 1);
        tc::mbar_init(&mma_done[0], 1);
        tc::mbar_init(&mma_done[1], 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(p.kch4 * WT_CHUNK_BYTES));
            for (int kc = 0; kc < p.kch4; ++kc)
                tc::tma_load_2d(sWT + kc * WT_CHUNK_BYTES, &p.map_wt, w_full, 64 * kc, j0);
            uint32_t stage = 0, phase = 0;
            bool aborted = false;
            // MMA iteration i = 1..T consumes dG_{T-i}, written in iteration i-1
            for (int i = 1; i <= T && !aborted; ++i) {
                if (!wait_counter(ctr, (unsigned)(p.S * i), p.ctrl, abort_flag, 0x301, p.wait_ns)) {
                    aborted = true;
                    break;
                }
                // acquire above, then the proxy fence: the TMA reads below see
                // every dG store the group released
                tc::fence_proxy_async_global();
                const int row0 = (T - i) * B + b0;
                int kc = rot;
                for (int ic = 0; ic < p.kch4; ++ic, kc = (kc + 1 == p.kch4) ? 0 : kc + 1) {
                    if (!tc::mbar_wait(&empty[stage], phase ^ 1, p.ctrl, abort_flag, 0x302,
                                       p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[stage], NB * 128);
                    tc::tma_load_2d(ring + stage * BWD_STAGE_BYTES, &p.map_dg, &full[stage], 64 * kc,
                                    row0);
                    if (++stage == (uint32_t)p.stages) stage = 0, phase ^= 1;
                }
            }
            if (aborted) {
                tc::mbar_wait(w_full, 0, nullptr, nullptr, 0, 200000000ull);
                for (int i = 0; i < p.stages; ++i) {
                    if (stage == 0) stage = p.stages, phase ^= 1;
                    --stage;
                    tc::mbar_wait(&full[stage], phase, nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            const uint32_t idesc = tc::idesc_bf16_f32(64, UNITS, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t r_lo0 = tc::smem_u32(ring) >> 4, w_lo0 = tc::smem_u32(sWT) >> 4;
            constexpr uint32_t RSTEP = BWD_STAGE_BYTES >> 4, WSTEP = WT_CHUNK_BYTES >> 4;
            bool ok = tc::mbar_wait(w_full, 0, p.ctrl, abort_flag, 0x303, p.wait_ns);
            for (int i = 1; ok && i <= T; ++i) {
                const uint32_t d = tmem_base + (i & 1) * UNITS;
                int kc = rot;
                for (int ic = 0; ic < p.kch4; ++ic, kc = (kc + 1 == p.kch4) ? 0 : kc + 1) {
                    if (!tc::mbar_wait(&full[stage], phase, p.ctrl, abort_flag, 0x304, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t ad = hi | (r_lo0 + stage * RSTEP);
                    const uint64_t bd = hi | (w_lo0 + kc * WSTEP);
                    tc::mma_bf16(d, ad, bd, idesc, ic != 0);
                    tc::mma_bf16(d, ad + 2, bd + 2, idesc, 1);
                    tc::mma_bf16(d, ad + 4, bd + 4, idesc, 1);
                    tc::mma_bf16(d, ad + 6, bd + 6, idesc, 1);
                    tc::mma_commit(&empty[stage]);
                    if (++stage == (uint32_t)p.stages) stage = 0, phase ^= 1;
                }
                if (ok) tc::mma_commit(&mma_done[i & 1]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;
        const int q = warp & 3;
        const int m = 16 * q + (lane & 15);
        const int half = lane >> 4;
        const int b = b0 + m;
        const int jb = j0 + 8 * half;
        const bool valid = (m < NB) && (b < B);
        const long long G4 = 4LL * H;
        float dc[8], dbacc[4][8];
        float gv[4][8], ct[8], cp[8], dyv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            dc[u] = (valid && p.dcT) ? p.dcT[(long long)b * H + jb + u] : 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) dbacc[g][u] = 0.f;
        }
        // saved forward state of step t for this thread's 8 (row, unit) pairs
        auto load_step = [&](int t) {
            if (!valid) {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    ct[u] = cp[u] = dyv[u] = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) gv[g][u] = 0.f;
                }
                return;
            }
            const long long row = (long long)t * B + b;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.gates + row * G4 + g * H + jb)),
                              gv[g]);
            const float4 *c4 = reinterpret_cast<const float4 *>(p.cells + row * H + jb);
            const float4 x0 = __ldg(c4), x1 = __ldg(c4 + 1);
            ct[0] = x0.x; ct[1] = x0.y; ct[2] = x0.z; ct[3] = x0.w;
            ct[4] = x1.x; ct[5] = x1.y; ct[6] = x1.z; ct[7] = x1.w;
            const float *cpp = t > 0 ? p.cells + (row - B) * H + jb
                                     : (p.c0 ? p.c0 + (long long)b * H + jb : nullptr);
            if (cpp) {
                const float4 y0 = __ldg(reinterpret_cast<const float4 *>(cpp));
                const float4 y1 = __ldg(reinterpret_cast<const float4 *>(cpp) + 1);
                cp[0] = y0.x; cp[1] = y0.y; cp[2] = y0.z; cp[3] = y0.w;
                cp[4] = y1.x; cp[5] = y1.y; cp[6] = y1.z; cp[7] = y1.w;
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) cp[u] = 0.f;
            }
            if (p.dy) {
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.dy + row * H + jb)), dyv);
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) dyv[u] = 0.f;
            }
        };
        // delta h from the MMA of iteration i (accumulator i & 1), 8 units per thread
        uint32_t dphase[2] = {0, 0};
        auto read_dh = [&](int i, float (&dh)[8]) -> bool {
            const int acc = i & 1;
            const bool w =
                tc::mbar_wait(&mma_done[acc], dphase[acc], p.ctrl, abort_flag, 0x305, p.wait_ns);
            if (!epi_vote_all(w)) return false;
            dphase[acc] ^= 1;
            tc::tc_fence_after();
            uint32_t r[16];
            tc::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + acc * UNITS, r);
            tc::tmem_ld_wait();
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float hi = __shfl_sync(0xffffffffu, __uint_as_float(r[8 + u]), lane & 15);
                dh[u] = half ? hi : __uint_as_float(r[u]);
            }
            tc::tc_fence_before();
            return true;
        };

        load_step(T - 1);
        bool ok = true;
        for (int i = 0; i < T; ++i) {
            const int t = T - 1 - i;
            float dhr[8];
            if (i == 0) {
                if (valid && p.dhT) {
                    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.dhT + (long long)b * H + jb)),
                                  dhr);
                } else {
#pragma unroll
                    for (int u = 0; u < 8; ++u) dhr[u] = 0.f;
                }
            } else if (!read_dh(i, dhr)) {
                ok = false;
                break;
            }
            float dI[8], dF[8], dGg[8], dO[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float ig = gv[0][u], fg = gv[1][u], gg = gv[2][u], og = gv[3][u];
                const float dh = dyv[u] + dhr[u];                       // step 1
                const float tc_ = tanh_fast(ct[u]);
                const float dcv = dh * og * (1.f - tc_ * tc_) + dc[u];  // step 2
                dO[u] = dh * tc_ * og * (1.f - og);                     // step 3
                dGg[u] = dcv * ig * (1.f - gg * gg);
                dI[u] = dcv * gg * ig * (1.f - ig);
                dF[u] = dcv * cp[u] * fg * (1.f - fg);
                dc[u] = dcv * fg;                                       // step 5
            }
            if (valid) {
                __nv_bfloat16 *o = p.dG + ((long long)t * B + b) * G4 + jb;
                const uint4 vi = f32x8_to_bf16(dI), vf = f32x8_to_bf16(dF);
                const uint4 vg = f32x8_to_bf16(dGg), vo = f32x8_to_bf16(dO);
                *reinterpret_cast<uint4 *>(o) = vi;
                *reinterpret_cast<uint4 *>(o + H) = vf;
                *reinterpret_cast<uint4 *>(o + 2 * H) = vg;
                *reinterpret_cast<uint4 *>(o + 3 * H) = vo;
                // db (step 4) sums the stored (rounded) values, as dW does
                float ri[8], rf[8], rg[8], ro[8];
                bf16x8_to_f32(vi, ri); bf16x8_to_f32(vf, rf);
                bf16x8_to_f32(vg, rg); bf16x8_to_f32(vo, ro);
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    dbacc[0][u] += ri[u];
                    dbacc[1][u] += rf[u];
                    dbacc[2][u] += rg[u];
                    dbacc[3][u] += ro[u];
                }
            }
            named_bar(1, EPI_THREADS);
            if (et == 0 && (int)blockIdx.x != p.fault_skip_cta) {
                red_release_add(ctr, 1u);  // release: the step's stores, ordered by bar.sync
            }
            if (t > 0) load_step(t - 1);
        }
        float dh0v[8];
        ok = ok && read_dh(T, dh0v);  // uniform over the epilogue threads
        if (ok && valid) {
            float4 *o = reinterpret_cast<float4 *>(p.dh0 + (long long)b * H + jb);
            o[0] = make_float4(dh0v[0], dh0v[1], dh0v[2], dh0v[3]);
            o[1] = make_float4(dh0v[4], dh0v[5], dh0v[6], dh0v[7]);
            float4 *oc = reinterpret_cast<float4 *>(p.dc0 + (long long)b * H + jb);
            oc[0] = make_float4(dc[0], dc[1], dc[2], dc[3]);
            oc[1] = make_float4(dc[4], dc[5], dc[6], dc[7]);
        }
        // db partial of this CTA: sum over its rows, in a fixed order
        if (ok) {
            float *red = reinterpret_cast<float *>(ring);  // [64 rows][64 = 4 gates x 16 units]
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    red[m * 64 + g * 16 + 8 * half + u] = valid ? dbacc[g][u] : 0.f;
            named_bar(1, EPI_THREADS);
            if (et < 64) {
                float sum = 0.f;
                for (int r = 0; r < 64; ++r) sum += red[r * 64 + et];
                const int g = et / 16, u = et % 16;
                p.db_part[(long long)gi * G4 + (long long)g * H + j0 + u] = sum;
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// W_h^T [H][4H] from W [4H][H+I] (the K-major B operand of the backward kernel).
__global__ void transpose_wh(const __nv_bfloat16 *__restrict__ W, __nv_bfloat16 *__restrict__ WT,
                             int H, int I) {
    __shared__ __nv_bfloat16 tile[32][33];
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;  // rows of W (4H), columns (H)
    const int tx = threadIdx.x, ty = threadIdx.y;          // 32 x 8
    for (int k = ty; k < 32; k += 8) {
        const int r = r0 + k, c = c0 + tx;
        if (r < 4 * H && c < H) tile[k][tx] = W[(long long)r * (H + I) + c];
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
        const int c = c0 + k, r = r0 + tx;
        if (r < 4 * H && c < H) WT[(long long)c * 4 * H + r] = tile[tx][k];
    }
}

// The same transpose with 64 x 64 tiles and 16-byte accesses (8 elements):
// W [4H][H + I] -> WT [H][4H].  Needs H and I multiples of 8 and 16-byte
// aligned W and WT; the elements are moved as raw 16-bit values.  Loads: a
// quarter warp reads one 128-byte row segment of W; stores: a warp writes
// 16 bytes (8 consecutive 4H-indices) of 32 consecutive WT rows, reading 32
// consecutive elements of one tile row per element of its vector.
__global__ void __launch_bounds__(256) transpose_wh_v8(const uint16_t *__restrict__ W,
                                                     uint16_t *__restrict__ WT, int H, int I) {
    __shared__ __align__(16) uint16_t tile[64][72];  // 144-byte rows: 16-byte aligned
    const int r0 = blockIdx.y * 64, c0 = blockIdx.x * 64;  // rows of W (4H), columns (H)
    const int G4 = 4 * H;
    const long long ld = (long long)H + I;
    for (int v = threadIdx.x; v < 64 * 8; v += 256) {
        const int rr = v / 8, cv = (v % 8) * 8;
        const int r = r0 + rr, c = c0 + cv;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (r < G4 && c < H) val = *reinterpret_cast<const uint4 *>(W + (long long)r * ld + c);
        *reinterpret_cast<uint4 *>(&tile[rr][cv]) = val;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < 64 * 8; v += 256) {
        const int cc = v % 64, rv = (v / 64) * 8;
        const int c = c0 + cc, r = r0 + rv;
        if (c >= H || r >= G4) continue;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = (uint32_t)tile[rv + 2 * i][cc] | ((uint32_t)tile[rv + 2 * i + 1][cc] << 16);
        *reinterpret_cast<uint4 *>(WT + (long long)c * G4 + r) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace rec
}  // namespace lstm
