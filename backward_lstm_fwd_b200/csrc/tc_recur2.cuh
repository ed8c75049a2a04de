// tc_recur2.cuh -- cluster versions of the persistent recurrent kernels (bf16).
//
// Why clusters: one tcgen05.mma instruction costs a roughly fixed ~120 cycles
// to issue, whatever its M x N, so the time of one recurrent step is set by
// the number of MMA instructions each CTA issues per step (K / 16 per output
// tile).  These kernels split the contraction dimension K over the CTAs of a
// thread-block cluster and use the largest tiles the problem allows (M = 128),
// so every CTA issues 4-8x fewer instructions per step than a K-resident
// design; the partial tiles are then reduce-scattered through distributed
// shared memory (DSMEM) inside the cluster.
//
// Forward ("SingleLayerLstmGrad", forward-formula table):
//   cluster = KS CTAs sharing 32 hidden units (128 gate rows of W_h: gate-major,
//   row m = 32 * gate + unit) and one batch group of NB rows; CTA k of the
//   cluster holds W_h[rows, k*Kc .. (k+1)*Kc) (Kc = H / KS) resident and streams
//   h_{t-1}[batch, same K range].  Per step: M = 128, N = NB, K = Kc MMAs; the
//   128 x NB partial tile is reduce-scattered over batch columns (CTA k keeps
//   columns k*NB/KS ..), the four gates of each unit meet in shared memory, and
//   the epilogue applies the nonlinearities and the cell / hidden update.
// Backward (backward algorithm steps 1-3, 5, 6; step 4's db on the way):
//   cluster = 8 CTAs sharing 128 hidden units and one batch group of <= 128
//   rows; CTA k holds W_h[k*Kc .. (k+1)*Kc, units] (Kc = 4H / 8, from a W_h^T
//   copy) and streams dG_{t+1}[rows, same K range].  Per step: M = 128 (batch
//   rows), N = 128 (units), K = Kc MMAs; the partial tile is reduce-scattered
//   over units (CTA k keeps units 16k .. 16k+15), and each of eight epilogue
//   warps finishes one batch row x 8 units per thread of the pointwise step.
//   (Clusters of 8 at ~220 KB of shared memory: at most 15 are co-resident on
//   a B200, which 128 units per cluster respects for H <= 1024.)
//
// Synchronisation: inside a cluster, remote mbarrier arrivals (release.cluster)
// after the DSMEM stores; across the CTAs of a batch group, one release /
// acquire counter per step (bounded waits, as in tc_recur.cuh).
#pragma once

#include "tc_recur.cuh"

namespace lstm {
namespace rec2 {

using rec::BAR_BYTES;
using rec::EPI_THREADS;
using rec::NUM_THREADS;

constexpr int MAX_KCC = 16;  // K chunks (of 64) per CTA

template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 2 || N == 4 || N == 8 || N == 16 || N == 32, "column block");
    if constexpr (N == 2) {
        tc::tmem_ld2(taddr, r);
    } else if constexpr (N == 32) {
        tc::tmem_ld32(taddr, r);
    } else if constexpr (N == 16) {
        tc::tmem_ld16(taddr, r);
    } else if constexpr (N == 8) {
        tc::tmem_ld8(taddr, r);
    } else {
        tc::tmem_ld4(taddr, r);
    }
}

// Receive buffers are chunk-major: [source][chunk of VW columns][row][VW].
// Consecutive rows (= consecutive lanes) are consecutive VW-float vectors, so
// one warp-wide vector store moves a contiguous 32 * VW * 4 bytes and the
// matching vector reads are bank-conflict free.

// =========================================================================
// forward
// =========================================================================
constexpr int F_UNITS = 32;
constexpr int F_ROWS = 4 * F_UNITS;       // 128: the MMA's M
constexpr int F_WCHUNK = F_ROWS * 128;    // 16 KB: 128 rows x 64 K of W_h
constexpr int F_EPI_WARPS = 8;            // two warps per TMEM lane quarter
constexpr int F_EPI_THREADS = 32 * F_EPI_WARPS;
constexpr int F_THREADS = 64 + F_EPI_THREADS;

struct Fwd2Params {
    CUtensorMap map_w;   // W [4H][H+I], box {64, 32}
    CUtensorMap map_y;   // y [T*B][H], box {64, NB}
    CUtensorMap map_h0;  // h0 [B][H], box {64, NB}
    const float *Gx, *c0;
    __nv_bfloat16 *y, *gates, *hT;
    float *cells, *cT;
    Ctrl *ctrl;
    int T, B, H, R, G, kcc, has_h0;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// Partials for the other CTAs of the cluster are staged in `send` ([KS-1
// destinations][chunks][128 rows][VW], the layout of the receive buffers) and
// moved by bulk copies; `send` aliases the ring (idle between the step's last
// MMA and the next step's loads) when the ring is large enough.
struct Fwd2Smem {
    int w, ring, recv, xbuf, send, bars, total;
    __host__ __device__ Fwd2Smem(int kcc, int NB, int KS) {
        const int NBc = NB / KS;
        const int ring_bytes = kcc * NB * 128, part_bytes = (KS - 1) * NBc * F_ROWS * 4;
        w = 0;
        ring = kcc * F_WCHUNK;
        recv = ring + ring_bytes;
        xbuf = recv + part_bytes;
        send = ring_bytes >= part_bytes ? ring : xbuf + 4 * NBc * F_UNITS * 4;
        bars = (send == ring ? xbuf + 4 * NBc * F_UNITS * 4 : send + part_bytes);
        total = bars + BAR_BYTES;
    }
};

template <int NB, int KS>
__global__ void __launch_bounds__(F_THREADS, 1) fwd2_kernel(const __grid_constant__ Fwd2Params p) {
    constexpr int NBc = NB / KS;       // batch columns finalised by this CTA
    constexpr int NBh = NBc / 2;       // columns each of the two warps of a quarter moves
    constexpr int NP = (NBc + 7) / 8;  // (unit, batch) pairs per epilogue thread
    constexpr int VW = NBh >= 4 ? 4 : 2;  // floats per DSMEM store / receive chunk
    static_assert(NBc >= 4 && NBc % 4 == 0 && NBc <= 32, "columns per CTA");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Fwd2Smem L(p.kcc, NB, KS);
    uint8_t *sW = smem + L.w;
    uint8_t *ring = smem + L.ring;
    float *recv = (float *)(smem + L.recv);  // [KS-1 sources][NBc/VW chunks][128 rows][VW]
    float *xbuf = (float *)(smem + L.xbuf);  // [4 gates][NBc][32 units]
    float *send = (float *)(smem + L.send);  // [KS-1 destinations][NBc/VW][128 rows][VW]
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *full = bars;
    uint64_t *empty = bars + MAX_KCC;
    uint64_t *w_full = bars + 2 * MAX_KCC;
    uint64_t *mma_done = w_full + 1;  // [2]
    uint64_t *recv_full = w_full + 3;
    uint32_t *tmem_slot = (uint32_t *)(w_full + 4);
    volatile int *abort_flag = (volatile int *)(w_full + 5);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int rs = cid % p.R, gi = cid / p.R;
    const int u0 = rs * F_UNITS, b0 = gi * NB;
    const int H = p.H, B = p.B, kcc = p.kcc;
    const int kbase = (int)kpart * kcc * 64;
    unsigned int *ctr = &p.ctrl->bar[gi];
    const unsigned int group_ctas = (unsigned)(p.R * KS);
    constexpr uint32_t TMEM_COLS = (2 * NB < 32) ? 32 : 2 * NB;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kcc; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(w_full, 1);
        tc::mbar_init(&mma_done[0], 1);
        tc::mbar_init(&mma_done[1], 1);
        tc::mbar_init(recv_full, 1);  // one local arrival (with the expected bytes) per step
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();  // every CTA's barriers exist before any remote arrival
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(kcc * F_WCHUNK));
            for (int c = 0; c < kcc; ++c)
                for (int g = 0; g < 4; ++g)
                    tc::tma_load_2d(sW + c * F_WCHUNK + g * F_UNITS * 128, &p.map_w, w_full,
                                    kbase + 64 * c, g * H + u0);
            uint32_t ph = 0;  // every step uses each ring slot once
            bool aborted = false;
            for (int t = 0; t < p.T && !aborted; ++t) {
                if (t > 0) {
                    if (!rec::wait_counter(ctr, group_ctas * (unsigned)t, p.ctrl, abort_flag, 0x401,
                                           p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    // the group's generic-proxy stores were released to this
                    // thread's acquire; order the TMA (async-proxy) reads after it
                    tc::fence_proxy_async_global();
                } else if (!p.has_h0) {
                    continue;
                }
                const CUtensorMap *m = t > 0 ? &p.map_y : &p.map_h0;
                const int row0 = t > 0 ? (t - 1) * B + b0 : b0;
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&empty[c], ph ^ 1, p.ctrl, abort_flag, 0x402, p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[c], NB * 128);
                    tc::tma_load_2d(ring + c * NB * 128, m, &full[c], kbase + 64 * c, row0);
                }
                ph ^= 1;
            }
            if (aborted) {  // let issued copies land before the CTA can exit
                tc::mbar_wait(w_full, 0, nullptr, nullptr, 0, 200000000ull);
                for (int c = 0; c < kcc; ++c)
                    tc::mbar_wait(&full[c], ph ^ 1, nullptr, nullptr, 0, 200000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(F_ROWS, NB, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t w_lo0 = tc::smem_u32(sW) >> 4, r_lo0 = tc::smem_u32(ring) >> 4;
            constexpr uint32_t WSTEP = F_WCHUNK >> 4, RSTEP = (NB * 128) >> 4;
            uint32_t ph = 0;
            bool ok = tc::mbar_wait(w_full, 0, p.ctrl, abort_flag, 0x403, p.wait_ns);
            for (int t = 0; ok && t < p.T; ++t) {
                const int acc = t & 1;
                if (t == 0 && !p.has_h0) {
                    tc::mbar_arrive(&mma_done[acc]);
                    continue;
                }
                const uint32_t d = tmem_base + acc * NB;
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&full[c], ph, p.ctrl, abort_flag, 0x404, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t ad = hi | (w_lo0 + c * WSTEP);
                    const uint64_t bd = hi | (r_lo0 + c * RSTEP);
                    tc::mma_bf16(d, ad, bd, idesc, c != 0);
                    tc::mma_bf16(d, ad + 2, bd + 2, idesc, 1);
                    tc::mma_bf16(d, ad + 4, bd + 4, idesc, 1);
                    tc::mma_bf16(d, ad + 6, bd + 6, idesc, 1);
                    tc::mma_commit(&empty[c]);
                }
                ph ^= 1;
                if (ok) tc::mma_commit(&mma_done[acc]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;  // 0..255
        const int q = warp & 3;           // TMEM lane quarter = gate of the row read
        const int hh = (warp - 2) >> 2;   // which half of each column block it moves
        const int mrow = 32 * q + lane;   // row of the partial tile: gate q, unit lane
        const int bc0 = b0 + (int)kpart * NBc;  // first batch row finalised here
        constexpr uint32_t PART_BYTES = NBc * F_ROWS * 4;  // one partner's partial tile
        // position of destination d among this CTA's partners (its send block),
        // and of this CTA among d's sources (its receive slot at d)
        auto dst_pos = [&](int d) { return d < (int)kpart ? d : d - 1; };
        auto src_slot = [&](int d) { return (int)kpart < d ? (int)kpart : (int)kpart - 1; };
        // pointwise pairs of this thread: pair index et + 256 k -> unit, column
        float c[NP], gx[4][NP];
        auto pair_unit = [&](int k) { return (et + F_EPI_THREADS * k) & 31; };
        auto pair_col = [&](int k) { return (et + F_EPI_THREADS * k) >> 5; };
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            const int n = pair_col(k), b = bc0 + n, j = u0 + pair_unit(k);
            c[k] = (p.c0 && n < NBc && b < B) ? p.c0[(long long)b * H + j] : 0.f;
        }
        auto load_gx = [&](int t) {
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int n = pair_col(k), b = bc0 + n, j = u0 + pair_unit(k);
                const bool v = n < NBc && b < B;
                const float *row = p.Gx + ((long long)t * B + b) * 4 * H + j;
#pragma unroll
                for (int g = 0; g < 4; ++g) gx[g][k] = v ? __ldg(row + g * H) : 0.f;
            }
        };
        load_gx(0);
        uint32_t dph[2] = {0, 0}, rph = 0;
        for (int t = 0; t < p.T; ++t) {
            const int acc = t & 1;
            const bool w = tc::mbar_wait(&mma_done[acc], dph[acc], p.ctrl, abort_flag, 0x405,
                                         p.wait_ns);
            if (!rec::epi_vote_all_n<F_EPI_THREADS>(w)) break;
            dph[acc] ^= 1;
            tc::tc_fence_after();
            if (t == 0 && !p.has_h0) {
#pragma unroll
                for (int n = 0; n < NBh; ++n) xbuf[(q * NBc + hh * NBh + n) * F_UNITS + lane] = 0.f;
            } else {
                float own[NBh];
#pragma unroll
                for (int d = 0; d < KS; ++d) {
                    uint32_t v[NBh];
                    tmem_ld_cols<NBh>(
                        tmem_base + ((uint32_t)(32 * q) << 16) + acc * NB + d * NBc + hh * NBh, v);
                    tc::tmem_ld_wait();
                    if (d == (int)kpart) {
#pragma unroll
                        for (int n = 0; n < NBh; ++n) own[n] = __uint_as_float(v[n]);
                    } else {
                        float *blk = send + dst_pos(d) * (PART_BYTES / 4);
#pragma unroll
                        for (int k = 0; k < NBh / VW; ++k) {
                            const int ch = hh * (NBh / VW) + k;
                            float *a = blk + (ch * F_ROWS + mrow) * VW;
                            if constexpr (VW == 4)
                                *reinterpret_cast<float4 *>(a) =
                                    make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                                __uint_as_float(v[4 * k + 2]),
                                                __uint_as_float(v[4 * k + 3]));
                            else
                                *reinterpret_cast<float2 *>(a) =
                                    make_float2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                        }
                    }
                }
                tc::tc_fence_before();
                if (KS > 1) {
                    // staged partials -> async proxy -> one bulk copy per partner,
                    // completing on the partner's receive barrier
                    tc::fence_proxy_async_smem();
                    rec::named_bar(1, F_EPI_THREADS);
                    if (et == 0) {
                        tc::mbar_arrive_expect_tx(recv_full, (KS - 1) * PART_BYTES);
                        const uint32_t recv_lo = tc::smem_u32(recv), bar_lo = tc::smem_u32(recv_full);
                        // rank kpart + s first: each CTA receives from one
                        // sender at a time instead of all sending to rank 0
#pragma unroll
                        for (int s = 1; s < KS; ++s) {
                            const int d = ((int)kpart + s) % KS;
                            tc::bulk_copy_to_peer(
                                tc::map_rank(recv_lo + (uint32_t)src_slot(d) * PART_BYTES, (uint32_t)d),
                                send + dst_pos(d) * (PART_BYTES / 4), PART_BYTES,
                                tc::map_rank(bar_lo, (uint32_t)d));
                        }
                        tc::bulk_commit();
                    }
                    const bool w2 = tc::mbar_wait_cluster(recv_full, rph, p.ctrl, abort_flag, 0x406,
                                                          p.wait_ns);
                    if (!rec::epi_vote_all_n<F_EPI_THREADS>(w2)) break;
                    rph ^= 1;
                }
#pragma unroll
                for (int sl = 0; sl < KS - 1; ++sl) {
                    const float *src = recv + sl * F_ROWS * NBc;
#pragma unroll
                    for (int k = 0; k < NBh / VW; ++k) {
                        const int ch = hh * (NBh / VW) + k;
                        if constexpr (VW == 4) {
                            const float4 x = *reinterpret_cast<const float4 *>(src + (ch * F_ROWS + mrow) * 4);
                            own[4 * k] += x.x;
                            own[4 * k + 1] += x.y;
                            own[4 * k + 2] += x.z;
                            own[4 * k + 3] += x.w;
                        } else {
                            const float2 x = *reinterpret_cast<const float2 *>(src + (ch * F_ROWS + mrow) * 2);
                            own[2 * k] += x.x;
                            own[2 * k + 1] += x.y;
                        }
                    }
                }
#pragma unroll
                for (int n = 0; n < NBh; ++n) xbuf[(q * NBc + hh * NBh + n) * F_UNITS + lane] = own[n];
            }
            rec::named_bar(1, F_EPI_THREADS);
            __nv_bfloat16 *yt = p.y + (long long)t * B * H;
            __nv_bfloat16 *gt = p.gates + (long long)t * B * 4 * H;
            float *ct = p.cells + (long long)t * B * H;
            float gsave[4][NP];
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int n = pair_col(k), uu = pair_unit(k);
                if (n >= NBc) continue;
                const int b = bc0 + n, j = u0 + uu;
                const float ig = rec::sigmoid_fast(xbuf[(0 * NBc + n) * F_UNITS + uu] + gx[0][k]);
                const float fg = rec::sigmoid_fast(xbuf[(1 * NBc + n) * F_UNITS + uu] + gx[1][k]);
                const float gg = rec::tanh_fast(xbuf[(2 * NBc + n) * F_UNITS + uu] + gx[2][k]);
                const float og = rec::sigmoid_fast(xbuf[(3 * NBc + n) * F_UNITS + uu] + gx[3][k]);
                c[k] = fg * c[k] + ig * gg;
                const float h = og * rec::tanh_fast(c[k]);
                gsave[0][k] = ig; gsave[1][k] = fg; gsave[2][k] = gg; gsave[3][k] = og;
                if (b < B) {
                    const long long o = (long long)b * H + j;
                    yt[o] = __float2bfloat16_rn(h);  // h_t: what the other CTAs wait for
                    if (t == p.T - 1) {
                        p.hT[o] = __float2bfloat16_rn(h);
                        p.cT[o] = c[k];
                    }
                }
            }
            rec::named_bar(1, F_EPI_THREADS);  // y[t] stored; xbuf and recv free again
            if (et == 0) {
                // the staging block (the ring) must be read out before this
                // CTA's arrival lets the next step's TMA refill the ring
                if (KS > 1) tc::bulk_wait_read_all();
                if ((int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr, 1u);
            }
            // saved state for the backward pass: not needed by the other CTAs
            // during the recurrence, so stored after the arrival (outside the
            // writes its release has to cover)
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int n = pair_col(k), uu = pair_unit(k);
                const int b = bc0 + n, j = u0 + uu;
                if (n >= NBc || b >= B) continue;
                ct[(long long)b * H + j] = c[k];
                __nv_bfloat16 *g4 = gt + (long long)b * 4 * H + j;
                g4[0] = __float2bfloat16_rn(gsave[0][k]);
                g4[H] = __float2bfloat16_rn(gsave[1][k]);
                g4[2 * H] = __float2bfloat16_rn(gsave[2][k]);
                g4[3 * H] = __float2bfloat16_rn(gsave[3][k]);
            }
            if (t + 1 < p.T) load_gx(t + 1);
        }
        if (et == 0) tc::bulk_wait_all();  // no copy of this CTA still in flight at exit
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();  // no partner may still be writing into this CTA's smem
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

// =========================================================================
// backward
// =========================================================================
constexpr int B_KS = 8;                    // cluster size: CTAs splitting 4H
constexpr int B_UNITS = 128;               // units per cluster (the MMA's N)
constexpr int B_UPC = B_UNITS / B_KS;      // units finalised per CTA: 16
constexpr int B_MROWS = 128;               // batch rows per tile (the MMA's M)
constexpr int B_WCHUNK = B_UNITS * 128;    // 16 KB: 128 units x 64 K of W_h^T
constexpr int B_ACHUNK = B_MROWS * 128;    // 16 KB: 128 rows x 64 K of dG
constexpr int B_EPI_WARPS = 8;             // two warps per TMEM lane quarter
constexpr int B_EPI_THREADS = 32 * B_EPI_WARPS;
constexpr int B_THREADS = 64 + B_EPI_THREADS;
constexpr int B_ROUND0 = 4;                                   // partners in the first exchange round
constexpr int B_PART_BYTES = B_UPC * B_MROWS * 4;             // one partner's partial: 8 KB
constexpr int B_STAGE_BYTES = B_ROUND0 * B_PART_BYTES;        // ring bytes the exchange stages

struct Bwd2Params {
    CUtensorMap map_wt;  // W_h^T [H][4H], box {64, 128}
    CUtensorMap map_dg;  // dG [T*B][4H], box {64, NBr}
    const __nv_bfloat16 *dy, *dhT, *gates;
    const float *dcT, *cells, *c0;
    __nv_bfloat16 *dG;
    float *dh0, *dc0, *db_part;
    Ctrl *ctrl;
    int T, B, H, U, G, NBr, kcc, stages;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

struct Bwd2Smem {
    int wt, ring, recv, bars, total;
    __host__ __device__ Bwd2Smem(int kcc, int stages) {
        wt = 0;
        ring = kcc * B_WCHUNK;
        recv = ring + stages * B_ACHUNK;
        bars = recv + (B_KS - 1) * B_UPC * B_MROWS * 4;
        total = bars + BAR_BYTES;
    }
};

__global__ void __launch_bounds__(B_THREADS, 1) bwd2_kernel(const __grid_constant__ Bwd2Params p) {
    constexpr int KS = B_KS, UPC = B_UPC, UPT = 8;  // UPT: units per epilogue thread
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Bwd2Smem L(p.kcc, p.stages);
    uint8_t *sWT = smem + L.wt;
    uint8_t *ring = smem + L.ring;
    float *recv = (float *)(smem + L.recv);  // [KS-1 sources][4 chunks][128 rows][4 units]
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *full = bars;
    uint64_t *empty = bars + MAX_KCC;
    uint64_t *w_full = bars + 2 * MAX_KCC;
    uint64_t *mma_done = w_full + 1;
    uint64_t *recv_full = w_full + 3;
    uint32_t *tmem_slot = (uint32_t *)(w_full + 4);
    volatile int *abort_flag = (volatile int *)(w_full + 5);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int us = cid % p.U, gi = cid / p.U;
    const int j0 = us * B_UNITS, b0 = gi * p.NBr;
    const int H = p.H, B = p.B, T = p.T, kcc = p.kcc, NBr = p.NBr, stages = p.stages;
    const int kbase = (int)kpart * kcc * 64;  // this CTA's part of the 4H axis
    unsigned int *ctr = &p.ctrl->bar[gi];
    const unsigned int group_ctas = (unsigned)(p.U * KS);
    constexpr uint32_t TMEM_COLS = 2 * B_UNITS;  // two 128-column accumulators

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(w_full, 1);
        tc::mbar_init(&mma_done[0], 1);
        tc::mbar_init(&mma_done[1], 1);
        tc::mbar_init(recv_full, 1);  // one local arrival (with the expected bytes) per step
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t a_bytes = (uint32_t)NBr * 128;  // rows loaded per chunk (NBr % 16 == 0)

    if (warp == 0) {
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(w_full, (uint32_t)(kcc * B_WCHUNK));
            for (int c = 0; c < kcc; ++c)
                tc::tma_load_2d(sWT + c * B_WCHUNK, &p.map_wt, w_full, kbase + 64 * c, j0);
            uint32_t stage = 0, ph = 0;
            bool aborted = false;
            // MMA iteration i = 1..T consumes dG_{T-i}, written in iteration i-1
            for (int i = 1; i <= T && !aborted; ++i) {
                if (!rec::wait_counter(ctr, group_ctas * (unsigned)i, p.ctrl, abort_flag, 0x501,
                                       p.wait_ns)) {
                    aborted = true;
                    break;
                }
                // acquire above, then the proxy fence: the TMA reads below see
                // every dG store the group released
                tc::fence_proxy_async_global();
                const int row0 = (T - i) * B + b0;
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&empty[stage], ph ^ 1, p.ctrl, abort_flag, 0x502, p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[stage], a_bytes);
                    tc::tma_load_2d(ring + stage * B_ACHUNK, &p.map_dg, &full[stage], kbase + 64 * c,
                                    row0);
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
            }
            if (aborted) {
                tc::mbar_wait(w_full, 0, nullptr, nullptr, 0, 200000000ull);
                for (int i = 0; i < stages; ++i) {
                    if (stage == 0) stage = stages, ph ^= 1;
                    --stage;
                    tc::mbar_wait(&full[stage], ph, nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_bf16_f32(B_MROWS, B_UNITS, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t r_lo0 = tc::smem_u32(ring) >> 4, w_lo0 = tc::smem_u32(sWT) >> 4;
            constexpr uint32_t RSTEP = B_ACHUNK >> 4, WSTEP = B_WCHUNK >> 4;
            uint32_t stage = 0, ph = 0;
            bool ok = tc::mbar_wait(w_full, 0, p.ctrl, abort_flag, 0x503, p.wait_ns);
            for (int i = 1; ok && i <= T; ++i) {
                const uint32_t d = tmem_base + (i & 1) * B_UNITS;
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&full[stage], ph, p.ctrl, abort_flag, 0x504, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t ad = hi | (r_lo0 + stage * RSTEP);
                    const uint64_t bd = hi | (w_lo0 + c * WSTEP);
                    tc::mma_bf16(d, ad, bd, idesc, c != 0);
                    tc::mma_bf16(d, ad + 2, bd + 2, idesc, 1);
                    tc::mma_bf16(d, ad + 4, bd + 4, idesc, 1);
                    tc::mma_bf16(d, ad + 6, bd + 6, idesc, 1);
                    tc::mma_commit(&empty[stage]);
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
                if (ok) tc::mma_commit(&mma_done[i & 1]);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;     // 0..255
        const int q = warp & 3;              // TMEM lane quarter: batch rows 32q..32q+31
        const int hh = (warp - 2) >> 2;      // which 8 of the CTA's 16 units
        const int m = 32 * q + lane;         // batch row of the tile = TMEM lane
        const int b = b0 + m;
        const bool valid = (m < NBr) && (b < B);
        const int uo = 8 * hh;               // offset of this thread's units within the 16
        const int jb = j0 + (int)kpart * UPC + uo;
        const long long G4 = 4LL * H;
        // Partials for the seven partners are staged in the ring (idle between
        // the last MMA of an iteration and the next iteration's loads) and sent
        // by bulk copies in two rounds (4 + 3 partners, 8 KB each): the ring
        // holds 32 KB.  Receive slots are per source, so sums are deterministic.
        constexpr uint32_t PART_BYTES = B_PART_BYTES;  // one partner's 16 units
        constexpr int ROUND0 = B_ROUND0;
        float *stage = reinterpret_cast<float *>(ring);
        // partners are served in the order kpart + 1, kpart + 2, ... so each
        // CTA receives from one sender at a time; src_slot(d): this CTA's
        // receive slot at d
        auto src_slot = [&](int d) { return (int)kpart < d ? (int)kpart : (int)kpart - 1; };
        const uint32_t recv_lo = tc::smem_u32(recv), recvbar_lo = tc::smem_u32(recv_full);
        float dc[UPT], dbacc[4][UPT];
        float gv[4][UPT], ct[UPT], cp[UPT], dyv[UPT];
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            dc[u] = (valid && p.dcT) ? p.dcT[(long long)b * H + jb + u] : 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) dbacc[g][u] = 0.f;
        }
        auto load_step = [&](int t) {
            if (!valid) {
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    ct[u] = cp[u] = dyv[u] = 0.f;
#pragma unroll
                    for (int g = 0; g < 4; ++g) gv[g][u] = 0.f;
                }
                return;
            }
            const long long row = (long long)t * B + b;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                rec::bf16x8_to_f32(
                    __ldg(reinterpret_cast<const uint4 *>(p.gates + row * G4 + g * H + jb)), gv[g]);
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
                for (int u = 0; u < UPT; ++u) cp[u] = 0.f;
            }
            if (p.dy) {
                rec::bf16x8_to_f32(__ldg(reinterpret_cast<const uint4 *>(p.dy + row * H + jb)), dyv);
            } else {
#pragma unroll
                for (int u = 0; u < UPT; ++u) dyv[u] = 0.f;
            }
        };
        // delta h of this thread's row and 8 units from MMA iteration i: own
        // part from TMEM plus the seven partners' parts received over DSMEM
        uint32_t dph[2] = {0, 0}, rph = 0;
        auto read_dh = [&](int i, float (&dh)[UPT]) -> bool {
            const int acc = i & 1;
            const bool w =
                tc::mbar_wait(&mma_done[acc], dph[acc], p.ctrl, abort_flag, 0x505, p.wait_ns);
            if (!rec::epi_vote_all_n<B_EPI_THREADS>(w)) return false;
            dph[acc] ^= 1;
            tc::tc_fence_after();
            const uint32_t col0 = tmem_base + ((uint32_t)(32 * q) << 16) + acc * B_UNITS + uo;
            {   // own 8 units
                uint32_t v[UPT];
                tc::tmem_ld8(col0 + kpart * UPC, v);
                tc::tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < UPT; ++u) dh[u] = __uint_as_float(v[u]);
            }
#pragma unroll
            for (int round = 0; round < 2; ++round) {
                const int p0 = round ? ROUND0 : 0, p1 = round ? KS - 1 : ROUND0;
                if (round) {
                    // the first round's copies must have read the ring
                    if (et == 0) tc::bulk_wait_read_all();
                    rec::named_bar(1, B_EPI_THREADS);
                }
#pragma unroll
                for (int sp = p0; sp < p1; ++sp) {
                    const int d = ((int)kpart + 1 + sp) % KS;  // dst_pos(d) == sp
                    uint32_t v[UPT];
                    tc::tmem_ld8(col0 + d * UPC, v);
                    tc::tmem_ld_wait();
                    float *blk = stage + (sp - p0) * (PART_BYTES / 4);
#pragma unroll
                    for (int k = 0; k < 2; ++k)  // units uo + 4k .. +3: chunk uo/4 + k
                        *reinterpret_cast<float4 *>(blk + ((uo / 4 + k) * B_MROWS + m) * 4) =
                            make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                        __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                }
                tc::fence_proxy_async_smem();
                rec::named_bar(1, B_EPI_THREADS);
                if (et == 0) {
                    if (round == 0) tc::mbar_arrive_expect_tx(recv_full, (KS - 1) * PART_BYTES);
#pragma unroll
                    for (int sp = p0; sp < p1; ++sp) {
                        const int d = ((int)kpart + 1 + sp) % KS;
                        tc::bulk_copy_to_peer(
                            tc::map_rank(recv_lo + (uint32_t)src_slot(d) * PART_BYTES, (uint32_t)d),
                            stage + (sp - p0) * (PART_BYTES / 4), PART_BYTES,
                            tc::map_rank(recvbar_lo, (uint32_t)d));
                    }
                    tc::bulk_commit();
                }
            }
            tc::tc_fence_before();
            const bool w2 =
                tc::mbar_wait_cluster(recv_full, rph, p.ctrl, abort_flag, 0x506, p.wait_ns);
            if (!rec::epi_vote_all_n<B_EPI_THREADS>(w2)) return false;
            rph ^= 1;
#pragma unroll
            for (int sl = 0; sl < KS - 1; ++sl) {
                const float *src = recv + sl * B_MROWS * UPC;
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    const float4 x = *reinterpret_cast<const float4 *>(src + ((uo / 4 + k) * B_MROWS + m) * 4);
                    dh[4 * k] += x.x;
                    dh[4 * k + 1] += x.y;
                    dh[4 * k + 2] += x.z;
                    dh[4 * k + 3] += x.w;
                }
            }
            // partners refill recv only after the next group barrier, which
            // needs this CTA's next arrival: these reads are safe
            return true;
        };

        load_step(T - 1);
        bool ok = true;
        for (int i = 0; i < T; ++i) {
            const int t = T - 1 - i;
            float dhr[UPT];
            if (i == 0) {
                if (valid && p.dhT) {
                    rec::bf16x8_to_f32(
                        __ldg(reinterpret_cast<const uint4 *>(p.dhT + (long long)b * H + jb)), dhr);
                } else {
#pragma unroll
                    for (int u = 0; u < UPT; ++u) dhr[u] = 0.f;
                }
            } else if (!read_dh(i, dhr)) {
                ok = false;
                break;
            }
            float dI[UPT], dF[UPT], dGg[UPT], dO[UPT];
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                const float ig = gv[0][u], fg = gv[1][u], gg = gv[2][u], og = gv[3][u];
                const float dh = dyv[u] + dhr[u];                       // step 1
                const float tc_ = rec::tanh_fast(ct[u]);
                const float dcv = dh * og * (1.f - tc_ * tc_) + dc[u];  // step 2
                dO[u] = dh * tc_ * og * (1.f - og);                     // step 3
                dGg[u] = dcv * ig * (1.f - gg * gg);
                dI[u] = dcv * gg * ig * (1.f - ig);
                dF[u] = dcv * cp[u] * fg * (1.f - fg);
                dc[u] = dcv * fg;                                       // step 5
            }
            if (valid) {
                __nv_bfloat16 *o = p.dG + ((long long)t * B + b) * G4 + jb;
                const uint4 vi = rec::f32x8_to_bf16(dI), vf = rec::f32x8_to_bf16(dF);
                const uint4 vg = rec::f32x8_to_bf16(dGg), vo = rec::f32x8_to_bf16(dO);
                *reinterpret_cast<uint4 *>(o) = vi;
                *reinterpret_cast<uint4 *>(o + H) = vf;
                *reinterpret_cast<uint4 *>(o + 2 * H) = vg;
                *reinterpret_cast<uint4 *>(o + 3 * H) = vo;
                float ri[UPT], rf[UPT], rg[UPT], ro[UPT];  // db sums the stored values
                rec::bf16x8_to_f32(vi, ri);
                rec::bf16x8_to_f32(vf, rf);
                rec::bf16x8_to_f32(vg, rg);
                rec::bf16x8_to_f32(vo, ro);
#pragma unroll
                for (int u = 0; u < UPT; ++u) {
                    dbacc[0][u] += ri[u];
                    dbacc[1][u] += rf[u];
                    dbacc[2][u] += rg[u];
                    dbacc[3][u] += ro[u];
                }
            }
            rec::named_bar(1, B_EPI_THREADS);
            if (et == 0) {
                tc::bulk_wait_read_all();  // the ring is refilled after this arrival
                if ((int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr, 1u);
            }
            if (t > 0) load_step(t - 1);
        }
        float dh0v[UPT];
        ok = ok && read_dh(T, dh0v);  // uniform over the epilogue threads
        if (ok && valid) {
            float4 *o = reinterpret_cast<float4 *>(p.dh0 + (long long)b * H + jb);
            o[0] = make_float4(dh0v[0], dh0v[1], dh0v[2], dh0v[3]);
            o[1] = make_float4(dh0v[4], dh0v[5], dh0v[6], dh0v[7]);
            float4 *oc = reinterpret_cast<float4 *>(p.dc0 + (long long)b * H + jb);
            oc[0] = make_float4(dc[0], dc[1], dc[2], dc[3]);
            oc[1] = make_float4(dc[4], dc[5], dc[6], dc[7]);
        }
        if (et == 0) tc::bulk_wait_all();  // no copy of this CTA in flight from here on
        if (ok) {
            // db partial of this CTA: its 128 rows x (4 gates x 16 units), in a
            // fixed order.  recv is free: every partner's last copy completed on
            // the receive barrier this CTA just waited for.
            rec::named_bar(1, B_EPI_THREADS);
            float *red = recv;  // [128 rows][64]
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int u = 0; u < UPT; ++u)
                    red[m * 64 + g * UPC + uo + u] = valid ? dbacc[g][u] : 0.f;
            rec::named_bar(1, B_EPI_THREADS);
            if (et < 64) {
                float sum = 0.f;
                for (int r = 0; r < B_MROWS; ++r) sum += red[r * 64 + et];
                const int g = et / UPC, u = et % UPC;
                p.db_part[(long long)gi * G4 + (long long)g * H + j0 + (int)kpart * UPC + u] = sum;
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace rec2
}  // namespace lstm
