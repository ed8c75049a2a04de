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

// Wait until *ctr >= target (acquire).  Bounded by limit_ns of %globaltimer;
// on time-out record LSTM_ERR_TIMEOUT with `site` and raise the abort flag.
__device__ __forceinline__ bool wait_counter(const unsigned int *ctr, unsigned int target,
                                             Ctrl *ctrl, volatile int *abort_flag,
                                             uint32_t site, unsigned long long limit_ns) {
    if (ld_acquire_u32(ctr) >= target) return true;
    const uint64_t t0 = tc::globaltimer_ns();
    while (true) {
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
struct FwdSmem {
    int w, ring, xbuf, bars, total;
    __host__ __device__ FwdSmem(int kch, int stages, int NB) {
        w = 0;
        ring = kch * KCH_BYTES;
        xbuf = ring + stages * NB * 128;
        bars = xbuf + 4 * NB * UNITS * 4;
        total = bars + 256;
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
    uint64_t *empty = bars + 8;             // [stages]
    uint64_t *w_full = bars + 16;
    uint64_t *mma_done = bars + 17;         // [2]
    uint32_t *tmem_slot = (uint32_t *)(bars + 20);
    volatile int *abort_flag = (volatile int *)(bars + 21);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int s = blockIdx.x % p.S, gi = blockIdx.x / p.S;
    const int j0 = s * UNITS, b0 = gi * NB;
    const int H = p.H, B = p.B;
    unsigned int *ctr = &p.ctrl->bar[gi];
    constexpr uint32_t TMEM_COLS = (2 * NB < 32) ? 32 : 2 * NB;

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
                    tc::fence_proxy_async_global();
                } else if (!p.has_h0) {
                    continue;  // h_{-1} = 0: no MMA at t = 0
                }
                const CUtensorMap *m = t > 0 ? &p.map_y : &p.map_h0;
                const int row0 = t > 0 ? (t - 1) * B + b0 : b0;
                bool ok = true;
                for (int kc = 0; kc < p.kch; ++kc) {
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
            uint32_t stage = 0, phase = 0;
            const uint32_t idesc = tc::idesc_bf16_f32(MROWS, NB, 0, 0);
            bool ok = tc::mbar_wait(w_full, 0, p.ctrl, abort_flag, 0x203, p.wait_ns);
            for (int t = 0; ok && t < p.T; ++t) {
                const int acc = t & 1;
                if (t == 0 && !p.has_h0) {
                    tc::mbar_arrive(&mma_done[acc]);
                    continue;
                }
                const uint32_t d = tmem_base + acc * NB;
                for (int kc = 0; kc < p.kch; ++kc) {
                    if (!tc::mbar_wait(&full[stage], phase, p.ctrl, abort_flag, 0x204, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint32_t a = tc::smem_u32(sW + kc * KCH_BYTES);
                    const uint32_t b = tc::smem_u32(ring + stage * NB * 128);
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        tc::mma_bf16(d, tc::smem_desc_sw128(a + 32 * k, 16, 1024),
                                     tc::smem_desc_sw128(b + 32 * k, 16, 1024), idesc,
                                     (kc | k) != 0);
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
            if (!tc::mbar_wait(&mma_done[acc], (t >> 1) & 1, p.ctrl, abort_flag, 0x205, p.wait_ns))
                break;
            tc::tc_fence_after();
            const bool zero = (t == 0 && !p.has_h0);
            // TMEM rows of this warp: gate q, unit = lane (lanes 0..15)
#pragma unroll
            for (int c0 = 0; c0 < NB; c0 += 16) {
                uint32_t r[16];
                tc::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + acc * NB + c0, r);
                tc::tmem_ld_wait();
                if (lane < UNITS) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        xbuf[(q * NB + c0 + i) * UNITS + lane] = zero ? 0.f : __uint_as_float(r[i]);
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
                const float ig = sigmoidf_(xbuf[(0 * NB + n) * UNITS + u] + gx[0][k]);
                const float fg = sigmoidf_(xbuf[(1 * NB + n) * UNITS + u] + gx[1][k]);
                const float gg = tanhf_(xbuf[(2 * NB + n) * UNITS + u] + gx[2][k]);
                const float og = sigmoidf_(xbuf[(3 * NB + n) * UNITS + u] + gx[3][k]);
                c[k] = fg * c[k] + ig * gg;
                const float h = og * tanhf_(c[k]);
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
            tc::fence_proxy_async_global();  // y[t] is read next by TMA (async proxy)
            named_bar(1, EPI_THREADS);       // all of y[t] stored; xbuf free again
            if (et == 0 && (int)blockIdx.x != p.fault_skip_cta) {
                __threadfence();
                red_release_add(ctr, 1u);
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

}  // namespace rec
}  // namespace lstm
