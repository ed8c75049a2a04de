// Backward recurrence (bf16) with the recurrent weights resident in tensor
// memory.  "SingleLayerLstmGrad", backward pass, steps 1-6: per reverse time
// step, delta h = dG_{t+1} W_h (the K = 4H contraction) feeds the pointwise
// gradient of the cell, and the step's dG_t feeds the next contraction.
//
// Work split (same grid as the cluster kernel in tc_recur2.cuh): clusters of 8
// CTAs; a cluster owns 128 hidden units and one group of up to 128 batch rows;
// CTA k of the cluster contracts K-part k of the 4H axis (H/2 wide) and
// finalises 16 of the 128 units after a reduce-scatter over DSMEM.
//
// What differs from that kernel: the CTA's slice of W_h^T (128 units x H/2 of
// K, 128 KB of bf16) is the MMA's A operand in TMEM (tcgen05.mma with A from
// tensor memory), so the accumulator is [128 units (lanes)][batch (columns)]
// and shared memory is free for a ring that holds the whole dG K-slice of a
// step (every chunk load of a step in flight at once) and for one exchange
// round with all seven partners.
#pragma once
#include "tc_recur2.cuh"

namespace lstm {
namespace rec3 {

constexpr int KS = 8;                        // cluster size: CTAs splitting 4H
constexpr int UNITS = 128;                   // units per cluster: the MMA's M (TMEM lanes)
constexpr int UPC = UNITS / KS;              // units finalised per CTA: 16
constexpr int NMAX = 128;                    // batch rows per group: the MMA's N
constexpr int ACHUNK = NMAX * 128;           // ring stage: 128 rows x 64 K of dG (16 KB)
constexpr int EPI_WARPS = 8;                 // two warps per TMEM lane quarter
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int THREADS = 64 + EPI_THREADS;
constexpr int PART_BYTES = UPC * NMAX * 4;   // one source's partial for 16 units: 8 KB
constexpr uint32_t D_COL = 0;                // accumulator: columns 0 .. NBr-1
constexpr uint32_t W_COL = 128;              // W_h^T slice: columns 128 .. 128 + H/4 - 1
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_STAGES = 12;
constexpr int MIN_STAGES = (KS - 1) * PART_BYTES / ACHUNK + 1;  // the ring stages one exchange: 4

struct Bwd3Params {
    CUtensorMap map_dg;               // dG [T*B][4H] bf16, box {64, NBr}
    const __nv_bfloat16 *wt;          // W_h^T [H][4H] bf16
    const __nv_bfloat16 *dy, *dhT, *gates;
    const float *dcT, *cells, *c0;
    __nv_bfloat16 *dG;
    float *dh0, *dc0, *db_part;
    Ctrl *ctrl;
    int T, B, H, U, G, NBr, kcc, stages;
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// ring: stages x 16 KB (also the send staging: 7 x 8 KB, between a step's last
// MMA and the next step's loads); recv: [8 sources][16 units][128 rows] fp32,
// the CTA's own partial in its own slot.
struct Bwd3Smem {
    int ring, recv, bars, total;
    __host__ __device__ explicit Bwd3Smem(int stages) {
        ring = 0;
        recv = stages * ACHUNK;
        bars = recv + KS * PART_BYTES;
        total = bars + rec::BAR_BYTES;
    }
};

// float offset of (unit r of the 16, batch row n) in one 8 KB partial block:
// rows of 128 floats, 16-byte groups XOR-swizzled by r so that a warp writing
// 8 units' rows, or reading 32 batch rows of one unit, is bank-conflict free
__device__ __forceinline__ int part_off(int r, int n) {
    return r * NMAX + ((((n >> 2) ^ (r & 7)) << 2) | (n & 3));
}

__global__ void __launch_bounds__(THREADS, 1) bwd3_kernel(const __grid_constant__ Bwd3Params p) {
    constexpr int UPT = 8;  // units per epilogue thread in the pointwise part
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Bwd3Smem L(p.stages);
    uint8_t *ring = smem + L.ring;
    float *recv = (float *)(smem + L.recv);
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *full = bars;
    uint64_t *empty = bars + MAX_STAGES;
    uint64_t *w_ready = bars + 2 * MAX_STAGES;  // W_h^T slice written to TMEM
    uint64_t *mma_done = w_ready + 1;
    uint64_t *recv_full = w_ready + 2;
    uint32_t *tmem_slot = (uint32_t *)(w_ready + 3);
    volatile int *abort_flag = (volatile int *)(w_ready + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int us = cid % p.U, gi = cid / p.U;
    const int j0 = us * UNITS, b0 = gi * p.NBr;
    const int H = p.H, B = p.B, T = p.T, kcc = p.kcc, NBr = p.NBr, stages = p.stages;
    const int kslice = kcc * 64;              // this CTA's part of the 4H axis
    const int kbase = (int)kpart * kslice;
    unsigned int *ctr = &p.ctrl->bar[gi];
    const unsigned int group_ctas = (unsigned)(p.U * KS);

    if (threadIdx.x == 0) {
        for (int i = 0; i < stages; ++i) {
            tc::mbar_init(&full[i], 1);
            tc::mbar_init(&empty[i], 1);
        }
        tc::mbar_init(w_ready, EPI_THREADS);
        tc::mbar_init(mma_done, 1);
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
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, ph = 0;
            bool aborted = false;
            // MMA iteration i = 1..T consumes dG_{T-i}, written in iteration i-1
            for (int i = 1; i <= T && !aborted; ++i) {
                if (!rec::wait_counter(ctr, group_ctas * (unsigned)i, p.ctrl, abort_flag, 0x601,
                                       p.wait_ns)) {
                    aborted = true;
                    break;
                }
                // acquire above, then the proxy fence: the TMA reads below see
                // every dG store the group released
                tc::fence_proxy_async_global();
                const int row0 = (T - i) * B + b0;
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&empty[stage], ph ^ 1, p.ctrl, abort_flag, 0x602, p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(&full[stage], a_bytes);
                    tc::tma_load_2d(ring + stage * ACHUNK, &p.map_dg, &full[stage], kbase + 64 * c,
                                    row0);
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
            }
            if (aborted) {  // let issued copies land before the CTA can exit
                for (int i = 0; i < stages; ++i) {
                    if (stage == 0) stage = stages, ph ^= 1;
                    --stage;
                    tc::mbar_wait(&full[stage], ph, nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // D[128 units][NBr] (+)= W_h^T slice (TMEM) x dG chunk^T (smem, K-major)
            const uint32_t idesc = tc::idesc_bf16_f32(UNITS, NBr, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t r_lo0 = tc::smem_u32(ring) >> 4;
            constexpr uint32_t RSTEP = ACHUNK >> 4;
            const uint32_t d = tmem_base + D_COL, a0 = tmem_base + W_COL;
            uint32_t stage = 0, ph = 0;
            bool ok = tc::mbar_wait(w_ready, 0, p.ctrl, abort_flag, 0x603, p.wait_ns);
            tc::tc_fence_after();
            // One accumulator suffices: iteration i + 1 starts after the group
            // barrier, which needs this CTA's arrival, which follows the
            // epilogue's reads of iteration i's accumulator.
            for (int i = 1; ok && i <= T; ++i) {
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(&full[stage], ph, p.ctrl, abort_flag, 0x604, p.wait_ns)) {
                        ok = false;
                        break;
                    }
                    tc::tc_fence_after();
                    const uint64_t bd = hi | (r_lo0 + stage * RSTEP);
                    const uint32_t a = a0 + 32 * c;  // 64 K = 32 columns per chunk
                    tc::mma_bf16_ts(d, a, bd, idesc, c != 0);
                    tc::mma_bf16_ts(d, a + 8, bd + 2, idesc, 1);
                    tc::mma_bf16_ts(d, a + 16, bd + 4, idesc, 1);
                    tc::mma_bf16_ts(d, a + 24, bd + 6, idesc, 1);
                    tc::mma_commit(&empty[stage]);
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
                if (ok) tc::mma_commit(mma_done);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;  // 0..255
        const int q = warp & 3;           // TMEM lane quarter
        const int hh = (warp - 2) >> 2;   // which half of the columns this warp moves
        {
            // W_h^T rows j0 + 32q + lane, this warp's half of the K slice ->
            // TMEM lanes 32q + lane, two bf16 per column (lower K in the low half)
            const int u = 32 * q + lane;
            const __nv_bfloat16 *src =
                p.wt + (long long)(j0 + u) * (4LL * H) + kbase + hh * (kslice / 2);
            const uint32_t taddr =
                tmem_base + ((uint32_t)(32 * q) << 16) + W_COL + (uint32_t)(hh * (kslice / 4));
            for (int n = 0; n < kslice / 32; ++n) {
                const uint4 x0 = __ldg(reinterpret_cast<const uint4 *>(src + 16 * n));
                const uint4 x1 = __ldg(reinterpret_cast<const uint4 *>(src + 16 * n + 8));
                const uint32_t r[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                tc::tmem_st8(taddr + 8 * n, r);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(w_ready);
        }
        // pointwise part: batch row m, 8 of the CTA's 16 units
        const int m = 32 * q + lane;
        const int b = b0 + m;
        const bool valid = (m < NBr) && (b < B);
        const int uo = 8 * hh;
        const int jb = j0 + (int)kpart * UPC + uo;
        const long long G4 = 4LL * H;
        float *stage_buf = reinterpret_cast<float *>(ring);
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
        // delta h of row m, units uo..uo+7 from MMA iteration i: each thread
        // moves its accumulator row (one unit, 64 batch rows) to the block of
        // the CTA that finalises the unit (its own recv slot, or the send
        // staging), one bulk copy per partner, then the 8 slots are summed in
        // source order.
        uint32_t dph = 0, rph = 0;
        auto read_dh = [&](float (&dh)[UPT]) -> bool {
            const bool w = tc::mbar_wait(mma_done, dph, p.ctrl, abort_flag, 0x605, p.wait_ns);
            if (!rec::epi_vote_all_n<EPI_THREADS>(w)) return false;
            dph ^= 1;
            tc::tc_fence_after();
            {
                const int u = 32 * q + lane;  // accumulator lane = unit of the cluster's 128
                const int dst = u >> 4, r = u & (UPC - 1);
                float *blk = dst == (int)kpart
                                 ? recv + (int)kpart * (PART_BYTES / 4)
                                 : stage_buf + ((dst - (int)kpart - 1 + KS) % KS) * (PART_BYTES / 4);
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    uint32_t v[32];
                    tc::tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + D_COL +
                                      (uint32_t)(hh * 64 + 32 * s),
                                  v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int n = hh * 64 + 32 * s + 4 * k;
                        *reinterpret_cast<float4 *>(blk + part_off(r, n)) =
                            make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                        __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                    }
                }
            }
            tc::tc_fence_before();
            tc::fence_proxy_async_smem();
            rec::named_bar(1, EPI_THREADS);
            if (et == 0) {
                tc::mbar_arrive_expect_tx(recv_full, (KS - 1) * PART_BYTES);
                // partners kpart + 1, kpart + 2, ...: each CTA receives from
                // one sender at a time
#pragma unroll
                for (int sp = 0; sp < KS - 1; ++sp) {
                    const int d = ((int)kpart + 1 + sp) % KS;
                    tc::bulk_copy_to_peer(
                        tc::map_rank(recv_lo + kpart * (uint32_t)PART_BYTES, (uint32_t)d),
                        stage_buf + sp * (PART_BYTES / 4), PART_BYTES,
                        tc::map_rank(recvbar_lo, (uint32_t)d));
                }
                tc::bulk_commit();
            }
            const bool w2 = tc::mbar_wait_cluster(recv_full, rph, p.ctrl, abort_flag, 0x606,
                                                  p.wait_ns);
            if (!rec::epi_vote_all_n<EPI_THREADS>(w2)) return false;
            rph ^= 1;
#pragma unroll
            for (int u = 0; u < UPT; ++u) dh[u] = 0.f;
#pragma unroll
            for (int sl = 0; sl < KS; ++sl) {
                const float *src = recv + sl * (PART_BYTES / 4);
#pragma unroll
                for (int u = 0; u < UPT; ++u) dh[u] += src[part_off(uo + u, m)];
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
            } else if (!read_dh(dhr)) {
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
            rec::named_bar(1, EPI_THREADS);
            if (et == 0) {
                tc::bulk_wait_read_all();  // the ring is refilled after this arrival
                if ((int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr, 1u);
            }
            if (t > 0) load_step(t - 1);
        }
        float dh0v[UPT];
        ok = ok && read_dh(dh0v);  // uniform over the epilogue threads
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
            // db partial of this CTA: its rows x (4 gates x 16 units), in a
            // fixed order.  recv is free: every partner's last copy completed on
            // the receive barrier this CTA just waited for.
            rec::named_bar(1, EPI_THREADS);
            float *red = recv;  // [128 rows][64]
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int u = 0; u < UPT; ++u)
                    red[m * 64 + g * UPC + uo + u] = valid ? dbacc[g][u] : 0.f;
            rec::named_bar(1, EPI_THREADS);
            if (et < 64) {
                float sum = 0.f;
                for (int r = 0; r < NMAX; ++r) sum += red[r * 64 + et];
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

}  // namespace rec3
}  // namespace lstm
