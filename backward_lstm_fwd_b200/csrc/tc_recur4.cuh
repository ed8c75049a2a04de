// Backward recurrence with two decoupled batch streams ("SingleLayerLstmGrad",
// backward pass, steps 1-6: per reverse time step, delta h = dG_{t+1} W_h feeds
// the pointwise gradient of the cell, and the step's dG_t feeds the next
// contraction).
//
// The work split is that of bwd3_kernel (tc_recur3.cuh): clusters of 8 CTAs,
// a cluster owns 128 hidden units and one group of up to 128 batch rows, CTA
// k keeps its slice of W_h^T (128 units x 4H/8 of K) in tensor memory as the
// MMA's A operand and finalises 16 units after a reduce-scatter over DSMEM.
//
// What differs: the group's rows are two independent batch streams of up to
// 64 rows, and every stage of the step chain has its own agent per stream --
// a TMA producer warp, an MMA-issuing warp, a TMEM accumulator, a receive
// block, and an epilogue warpgroup -- with a group step counter per stream.
// A step of the chain is a global hand-off (release of the step's dG, the
// group counter, the TMA load of dG_{t+1}) followed by the contraction, the
// DSMEM exchange and the pointwise work; with the streams decoupled, one
// stream's hand-off and loads proceed while the other stream contracts,
// exchanges or computes, instead of every stage of the CTA waiting for the
// slowest stage of the other stream.
#pragma once
#include "tc_recur3.cuh"

namespace lstm {
namespace rec4 {

constexpr int KS = 8;                         // cluster size: CTAs splitting 4H
constexpr int UNITS = 128;                    // units per cluster: the MMA's M (TMEM lanes)
constexpr int UPC = UNITS / KS;               // units finalised per CTA: 16
constexpr int NSTREAM = 2;                    // batch streams per group
constexpr int NBS_MAX = 64;                   // rows per stream: the MMA's N
constexpr int CHUNK = NBS_MAX * 128;          // ring stage: 64 rows x 64 K of dG (8 KB)
constexpr int EPI_WG = 128;                   // epilogue threads per stream (one warp per lane quarter)
constexpr int THREADS = 128 + NSTREAM * EPI_WG;  // 4 agent warps + 2 epilogue warpgroups
constexpr int PART_BYTES = UPC * NBS_MAX * 4;    // one source's partial for 16 units: 4 KB
constexpr uint32_t W_COL = 128;               // W_h^T slice: columns 128 .. 128 + kcc*32 - 1
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_STAGES = 12;                // ring stages per stream
// the ring of a stream also stages its send blocks (7 x 4 KB) between the
// step's last MMA and the next step's loads
constexpr int MIN_STAGES = (KS - 1) * PART_BYTES / CHUNK + 1;  // 4

template <class E>  // E: the 16-bit compute type, __nv_bfloat16 or __half
struct Bwd4Params {
    CUtensorMap map_dg;               // dG [T*B][4H], box {64, NBS}
    const E *wt;                      // W_h^T [H][4H]
    const E *dy, *dhT, *gates;
    const float *dcT, *cells, *c0;
    E *dG;
    float *dh0, *dc0, *db_part;
    float *dc_carry;   // [B][H]: delta c between the launches of a chunked call
    const E *mask;     // variable length (MASKED): [T][B][H], 1 = real step
    float *dhp_carry;  // [B][H]: the delta h padding passes on, between launches
    Ctrl *ctrl;
    int T, B, H, U, G, NBr, NBS, kcc, stages;
    int i0, i1;        // this launch runs epilogue iterations i0 .. i1-1 (step T-1-i)
    int reverse;       // direction "REDIRECTIONAL": recurrence step s is at time T-1-s
    int bar_base;      // first of the call's G * NSTREAM step counters in ctrl->bar
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// Per stream: ring (stages x 8 KB, also the send staging), recv
// ([8 sources][16 units][64 rows] fp32, the CTA's own partial in its own slot).
struct Bwd4Smem {
    int ring[NSTREAM], recv[NSTREAM], red, bars, total;
    __host__ __device__ explicit Bwd4Smem(int stages) {
        int o = 0;
        for (int s = 0; s < NSTREAM; ++s) {
            ring[s] = o;
            o += stages * CHUNK;
            recv[s] = o;
            o += KS * PART_BYTES;
        }
        red = recv[0];  // the db reduction ([128 rows][64] fp32) reuses stream 0's recv block
        bars = o;
        total = bars + 1024;
    }
};

// float offset of (unit r of the 16, batch row n) in one 4 KB partial block:
// rows of 64 floats, 16-byte groups XOR-swizzled by r so that a warp writing
// 8 units' rows, or reading 32 batch rows of one unit, is bank-conflict free
__device__ __forceinline__ int part_off(int r, int n) {
    return r * NBS_MAX + ((((n >> 2) ^ (r & 7)) << 2) | (n & 3));
}

// MASKED: variable-length mask; IJFO: gate_order "ijfo"
template <class E, bool MASKED, bool IJFO>
__global__ void __launch_bounds__(THREADS, 1) bwd4_kernel(const __grid_constant__ Bwd4Params<E> p) {
    constexpr int UPT = 8;  // units per epilogue thread in the pointwise part
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const Bwd4Smem L(p.stages);
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    // per stream s: full[s][MAX_STAGES], empty[s][MAX_STAGES], mma_done[s], recv_full[s]
    auto full = [&](int s, int i) { return bars + s * 2 * MAX_STAGES + i; };
    auto empty = [&](int s, int i) { return bars + s * 2 * MAX_STAGES + MAX_STAGES + i; };
    uint64_t *w_ready = bars + NSTREAM * 2 * MAX_STAGES;  // W_h^T slice written to TMEM
    uint64_t *mma_done = w_ready + 1;                     // [NSTREAM]
    uint64_t *recv_full = w_ready + 1 + NSTREAM;          // [NSTREAM]
    uint64_t *xtok = w_ready + 1 + 2 * NSTREAM;           // [NSTREAM]: a stream's exchange is done
    uint32_t *tmem_slot = (uint32_t *)(w_ready + 1 + 3 * NSTREAM);
    volatile int *abort_flag = (volatile int *)(w_ready + 2 + 3 * NSTREAM);
    volatile int *cluster_bad = abort_flag + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int us = cid % p.U, gi = cid / p.U;
    const int j0 = us * UNITS, b0 = gi * p.NBr;
    const int H = p.H, B = p.B, T = p.T, kcc = p.kcc, NBS = p.NBS, stages = p.stages;
    const int i0 = p.i0, i1 = p.i1;
    const bool first = i0 == 0, last = i1 == T;
    const int mma_lo = i0 > 1 ? i0 : 1, mma_hi = last ? T : i1 - 1;
    auto tau = [&](int s) { return p.reverse ? T - 1 - s : s; };
    const int kslice = kcc * 64;  // this CTA's part of the 4H axis
    const int kbase = (int)kpart * kslice;
    const unsigned int group_ctas = (unsigned)(p.U * KS);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTREAM; ++s) {
            for (int i = 0; i < stages; ++i) {
                tc::mbar_init(full(s, i), 1);
                tc::mbar_init(empty(s, i), 1);
            }
            tc::mbar_init(&mma_done[s], 1);
            tc::mbar_init(&recv_full[s], 1);  // one local arrival (with the expected bytes) per step
            tc::mbar_init(&xtok[s], 1);
        }
        tc::mbar_init(w_ready, NSTREAM * EPI_WG);
        *abort_flag = 0;
        // the kernel is written for clusters of exactly KS CTAs
        *cluster_bad = tc::cluster_nctarank() != (uint32_t)KS;
        tc::fence_mbar_init();
    }
    if (warp == 2) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*cluster_bad) {  // a launch without the cluster shape: report, touch no peer
        if (threadIdx.x == 0) atomicCAS(&p.ctrl->status, 0u, 2u);  // LSTM_ERR_UNSUPPORTED
        if (warp == 2) {
            tc::tc_fence_after();
            tc::tmem_dealloc(*tmem_slot, TMEM_COLS);
        }
        return;
    }
    tc::cluster_sync_all();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp < 2) {
        // --------------------------------------------------- TMA producer of stream `warp`
        const int s = warp;
        if (lane == 0) {
            uint8_t *ring = smem + L.ring[s];
            unsigned int *ctr = &p.ctrl->bar[p.bar_base + gi * NSTREAM + s];
            const uint32_t bytes = (uint32_t)NBS * 128;
            uint32_t stage = 0, ph = 0;
            bool aborted = false;
            // MMA iteration i consumes dG_{T-i}, written in iteration i-1
            for (int i = mma_lo; i <= mma_hi && !aborted; ++i) {
                if (!rec::wait_counter(ctr, group_ctas * (unsigned)i, p.ctrl, abort_flag, 0x801,
                                       p.wait_ns)) {
                    aborted = true;
                    break;
                }
                // acquire above, then the proxy fence: the TMA reads below see
                // every dG store the group released
                tc::fence_proxy_async_global();
                const int row0 = tau(T - i) * B + b0 + s * NBS;  // this stream's rows of step T-i
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(empty(s, stage), ph ^ 1, p.ctrl, abort_flag, 0x802,
                                       p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    tc::mbar_arrive_expect_tx(full(s, stage), bytes);
                    tc::tma_load_2d(ring + stage * CHUNK, &p.map_dg, full(s, stage),
                                    kbase + 64 * c, row0);
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
            }
            if (aborted) {  // let issued copies land before the CTA can exit
                for (int i = 0; i < stages; ++i) {
                    if (stage == 0) stage = stages, ph ^= 1;
                    --stage;
                    tc::mbar_wait(full(s, stage), ph, nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp < 4) {
        // ------------------------------------------------------ MMA issuer of stream warp - 2
        const int s = warp - 2;
        if (lane == 0) {
            // D_s[128 units][NBS] (+)= W_h^T slice (TMEM) x dG chunk^T (smem, K-major)
            const uint32_t idesc = tc::idesc_f16kind_f32(Elem<E>::kFmt, UNITS, NBS, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t r_lo0 = tc::smem_u32(smem + L.ring[s]) >> 4;
            constexpr uint32_t RSTEP = CHUNK >> 4;
            const uint32_t d = tmem_base + (uint32_t)(s * NBS_MAX), a0 = tmem_base + W_COL;
            uint32_t stage = 0, ph = 0;
            bool ok = tc::mbar_wait(w_ready, 0, p.ctrl, abort_flag, 0x803, p.wait_ns);
            tc::tc_fence_after();
            // One accumulator per stream suffices: iteration i + 1 starts after
            // the stream's group barrier, which needs this CTA's arrival, which
            // follows the epilogue's reads of iteration i's accumulator.
            for (int i = mma_lo; ok && i <= mma_hi; ++i) {
                for (int c = 0; c < kcc; ++c) {
                    if (!tc::mbar_wait(full(s, stage), ph, p.ctrl, abort_flag, 0x804, p.wait_ns)) {
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
                    tc::mma_commit(empty(s, stage));
                    if (++stage == (uint32_t)stages) stage = 0, ph ^= 1;
                }
                if (ok) tc::mma_commit(&mma_done[s]);
            }
        }
    } else {
        // ------------------------------------------- epilogue warpgroup of stream sw
        const int et = threadIdx.x - 128;  // 0..255
        const int sw = et / EPI_WG;        // stream
        const int wt = et % EPI_WG;        // thread within the warpgroup
        const int q = warp & 3;            // TMEM lane quarter
        const int bar_sync = 1 + 2 * sw, bar_vote = 2 + 2 * sw;
        {
            // W_h^T rows j0 + 32q + lane, this warpgroup's half of the K slice
            // -> TMEM lanes 32q + lane, two elements per column (lower K in the low half)
            const int u = 32 * q + lane;
            const E *src = p.wt + (long long)(j0 + u) * (4LL * H) + kbase + sw * (kslice / 2);
            const uint32_t taddr = tmem_base + ((uint32_t)(32 * q) << 16) + W_COL +
                                   (uint32_t)(sw * (kslice / 4));
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
        float *recv = reinterpret_cast<float *>(smem + L.recv[sw]);
        float *stage_buf = reinterpret_cast<float *>(smem + L.ring[sw]);
        uint64_t *rf = &recv_full[sw];
        unsigned int *ctr = &p.ctrl->bar[p.bar_base + gi * NSTREAM + sw];
        // pointwise part: batch row m of the stream, 8 of the CTA's 16 units
        const int m = wt & (NBS_MAX - 1);
        const int uo = 8 * (wt / NBS_MAX);
        const int b = b0 + sw * NBS + m;
        const bool valid = (m < NBS) && (b < B);
        const int jb = j0 + (int)kpart * UPC + uo;
        const long long G4 = 4LL * H;
        const uint32_t recv_lo = tc::smem_u32(recv), recvbar_lo = tc::smem_u32(rf);
        float dc[UPT], dbacc[4][UPT];
        constexpr int kBlk[4] = {0, IJFO ? 2 : 1, IJFO ? 1 : 2, 3};
        uint4 gpk[4], dypk;  // prefetched gates and dy of the next step, still packed
        uint4 mpk;           // and its mask (MASKED)
        float ct[UPT], cp[UPT];
        float dhp[UPT];      // delta h that padding passes to h_{t-1} (MASKED)
#pragma unroll
        for (int u = 0; u < UPT; ++u) {
            const float *dcin = first ? p.dcT : p.dc_carry;
            dc[u] = (valid && dcin) ? dcin[(long long)b * H + jb + u] : 0.f;
            dhp[u] = (MASKED && !first && valid) ? p.dhp_carry[(long long)b * H + jb + u] : 0.f;
#pragma unroll
            for (int g = 0; g < 4; ++g) dbacc[g][u] = 0.f;
        }
        auto load_step = [&](int t) {
            if (!valid) {
#pragma unroll
                for (int u = 0; u < UPT; ++u) ct[u] = cp[u] = 0.f;
#pragma unroll
                for (int g = 0; g < 4; ++g) gpk[g] = make_uint4(0, 0, 0, 0);
                dypk = make_uint4(0, 0, 0, 0);
                mpk = make_uint4(0, 0, 0, 0);
                return;
            }
            const long long row = (long long)tau(t) * B + b;  // t: a step, not a time
#pragma unroll
            for (int g = 0; g < 4; ++g)
                gpk[g] = __ldg(reinterpret_cast<const uint4 *>(p.gates + row * G4 + kBlk[g] * H + jb));
            const float4 *c4 = reinterpret_cast<const float4 *>(p.cells + row * H + jb);
            const float4 x0 = __ldg(c4), x1 = __ldg(c4 + 1);
            ct[0] = x0.x; ct[1] = x0.y; ct[2] = x0.z; ct[3] = x0.w;
            ct[4] = x1.x; ct[5] = x1.y; ct[6] = x1.z; ct[7] = x1.w;
            const float *cpp = t > 0 ? p.cells + ((long long)tau(t - 1) * B + b) * H + jb
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
            dypk = p.dy ? __ldg(reinterpret_cast<const uint4 *>(p.dy + row * H + jb))
                        : make_uint4(0, 0, 0, 0);
            if (MASKED) mpk = __ldg(reinterpret_cast<const uint4 *>(p.mask + row * H + jb));
        };
        // delta h of row m, units uo..uo+7 from this stream's MMA iteration:
        // each thread moves its accumulator row (one unit, the stream's rows)
        // to the block of the CTA that finalises the unit (its own recv slot,
        // or the send staging), one bulk copy per partner, then the 8 slots
        // are summed in source order.
        // The two streams' DSMEM exchanges alternate: exchange k of stream 1
        // follows exchange k of stream 0, which follows exchange k - 1 of
        // stream 1.  Left free, the two symmetric chains fall into lockstep
        // and contend for the SM's DSMEM, TMA and memory bandwidth at the same
        // moments, settling into one of two step periods (the slower one 45 %
        // longer); offset only at the start of a launch they mostly stay
        // apart (2 % faster than strict alternation) but drifted into the slow
        // period in one run of 17.  Alternating, one stream's exchange runs
        // beside the other's hand-off, loads and pointwise work at every step.
        uint32_t dph = 0, rph = 0;
        int xk = 0;  // exchanges of this stream so far in this launch
        auto read_dh = [&](float (&dh)[UPT]) -> bool {
            const bool w = tc::mbar_wait(&mma_done[sw], dph, p.ctrl, abort_flag, 0x805, p.wait_ns);
            if (!rec3::vote_all(w, bar_vote, EPI_WG)) return false;
            dph ^= 1;
            tc::tc_fence_after();
            {
                const int u = 32 * q + lane;  // accumulator lane = unit of the cluster's 128
                const int dst = u >> 4, r = u & (UPC - 1);
                float *blk = dst == (int)kpart
                                 ? recv + (int)kpart * (PART_BYTES / 4)
                                 : stage_buf + ((dst - (int)kpart - 1 + KS) % KS) * (PART_BYTES / 4);
                const uint32_t tq = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(sw * NBS_MAX);
#pragma unroll
                for (int s4 = 0; s4 < NBS_MAX / 16; ++s4) {
                    if (16 * s4 >= NBS) break;  // warp-uniform
                    uint32_t v[16];
                    tc::tmem_ld16(tq + (uint32_t)(16 * s4), v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int n = 16 * s4 + 4 * k;
                        *reinterpret_cast<float4 *>(blk + part_off(r, n)) =
                            make_float4(__uint_as_float(v[4 * k]), __uint_as_float(v[4 * k + 1]),
                                        __uint_as_float(v[4 * k + 2]), __uint_as_float(v[4 * k + 3]));
                    }
                }
            }
            tc::tc_fence_before();
            tc::fence_proxy_async_smem();
            rec::named_bar(bar_sync, EPI_WG);
            if (wt == 0) {
                bool go = true;
                if (sw == 1)
                    go = tc::mbar_wait(&xtok[0], (uint32_t)(xk & 1), p.ctrl, abort_flag, 0x807,
                                       p.wait_ns);
                else if (xk > 0)
                    go = tc::mbar_wait(&xtok[1], (uint32_t)((xk - 1) & 1), p.ctrl, abort_flag,
                                       0x807, p.wait_ns);
                if (go) {
                    tc::mbar_arrive_expect_tx(rf, (KS - 1) * PART_BYTES);
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
            }
            const bool w2 = tc::mbar_wait_cluster(rf, rph, p.ctrl, abort_flag, 0x806, p.wait_ns);
            if (!rec3::vote_all(w2, bar_vote, EPI_WG)) return false;
            if (wt == 0) tc::mbar_arrive(&xtok[sw]);
            ++xk;
            rph ^= 1;
#pragma unroll
            for (int u = 0; u < UPT; ++u) dh[u] = 0.f;
#pragma unroll
            for (int sl = 0; sl < KS; ++sl) {
                const float *src = recv + sl * (PART_BYTES / 4);
#pragma unroll
                for (int u = 0; u < UPT; ++u) dh[u] += src[part_off(uo + u, m)];
            }
            // partners refill recv only after the stream's next group barrier,
            // which needs this CTA's next arrival: these reads are safe
            return true;
        };

        load_step(T - 1 - i0);
        bool ok = true;
        for (int i = i0; i < i1; ++i) {
            const int t = T - 1 - i;
            float dhr[UPT];
            if (i == 0) {
                if (valid && p.dhT) {
                    x8_to_f32<E>(
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
            float gv[4][UPT], dyv[UPT];
#pragma unroll
            for (int g = 0; g < 4; ++g) x8_to_f32<E>(gpk[g], gv[g]);
            x8_to_f32<E>(dypk, dyv);
            float mkv[UPT];
            if (MASKED) x8_to_f32<E>(mpk, mkv);
#pragma unroll
            for (int u = 0; u < UPT; ++u) {
                const float ig = gv[0][u], fg = gv[1][u], gg = gv[2][u], og = gv[3][u];
                float dh = dyv[u] + dhr[u];                             // step 1
                float dcn = dc[u], dc_pass = 0.f;
                if (MASKED) {  // padding: the share 1 - m passes to h_{t-1}, c_{t-1}
                    dh += dhp[u];
                    dhp[u] = __fmul_rn(1.f - mkv[u], dh);
                    dh = __fmul_rn(dh, mkv[u]);
                    dc_pass = __fmul_rn(1.f - mkv[u], dcn);
                    dcn = __fmul_rn(dcn, mkv[u]);
                }
                const float tc_ = rec::tanh_fast(ct[u]);
                const float dcv = dh * og * (1.f - tc_ * tc_) + dcn;    // step 2
                dO[u] = dh * tc_ * og * (1.f - og);                     // step 3
                dGg[u] = dcv * ig * (1.f - gg * gg);
                dI[u] = dcv * gg * ig * (1.f - ig);
                dF[u] = dcv * cp[u] * fg * (1.f - fg);
                dc[u] = dcv * fg + dc_pass;                             // step 5
            }
            {
                const uint4 vi = f32x8_to<E>(dI), vf = f32x8_to<E>(dF);
                const uint4 vg = f32x8_to<E>(dGg), vo = f32x8_to<E>(dO);
                if (valid) {
                    E *o = p.dG + ((long long)tau(t) * B + b) * G4 + jb;
                    *reinterpret_cast<uint4 *>(o) = vi;
                    *reinterpret_cast<uint4 *>(o + kBlk[1] * H) = vf;
                    *reinterpret_cast<uint4 *>(o + kBlk[2] * H) = vg;
                    *reinterpret_cast<uint4 *>(o + 3 * H) = vo;
                    float ri[UPT], rf_[UPT], rg[UPT], ro[UPT];  // db sums the stored values
                    x8_to_f32<E>(vi, ri);
                    x8_to_f32<E>(vf, rf_);
                    x8_to_f32<E>(vg, rg);
                    x8_to_f32<E>(vo, ro);
#pragma unroll
                    for (int u = 0; u < UPT; ++u) {
                        dbacc[0][u] += ri[u];
                        dbacc[1][u] += rf_[u];
                        dbacc[2][u] += rg[u];
                        dbacc[3][u] += ro[u];
                    }
                }
            }
            rec::named_bar(bar_sync, EPI_WG);
            if (wt == 0) {
                tc::bulk_wait_read_all();  // the ring is refilled after this arrival
                if ((int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr, 1u);
            }
            if (i + 1 < i1) load_step(t - 1);
        }
        float dh0v[UPT];
        if (!last) {
            if (ok && valid) {  // delta c (and delta h passed by padding) for the next launch
                float4 *oc = reinterpret_cast<float4 *>(p.dc_carry + (long long)b * H + jb);
                oc[0] = make_float4(dc[0], dc[1], dc[2], dc[3]);
                oc[1] = make_float4(dc[4], dc[5], dc[6], dc[7]);
                if (MASKED) {
                    float4 *oh = reinterpret_cast<float4 *>(p.dhp_carry + (long long)b * H + jb);
                    oh[0] = make_float4(dhp[0], dhp[1], dhp[2], dhp[3]);
                    oh[1] = make_float4(dhp[4], dhp[5], dhp[6], dhp[7]);
                }
            }
        } else {
            ok = ok && read_dh(dh0v);  // uniform over the warpgroup
            if (MASKED) {
#pragma unroll
                for (int u = 0; u < UPT; ++u) dh0v[u] += dhp[u];
            }
            if (ok && valid) {
                float4 *o = reinterpret_cast<float4 *>(p.dh0 + (long long)b * H + jb);
                o[0] = make_float4(dh0v[0], dh0v[1], dh0v[2], dh0v[3]);
                o[1] = make_float4(dh0v[4], dh0v[5], dh0v[6], dh0v[7]);
                float4 *oc = reinterpret_cast<float4 *>(p.dc0 + (long long)b * H + jb);
                oc[0] = make_float4(dc[0], dc[1], dc[2], dc[3]);
                oc[1] = make_float4(dc[4], dc[5], dc[6], dc[7]);
            }
        }
        if (wt == 0) tc::bulk_wait_all();  // no copy of this stream in flight from here on
        // db partial of this CTA: both streams' rows x (4 gates x 16 units),
        // in a fixed order.  Both recv blocks are free: every partner's last
        // copy completed on the receive barriers these warpgroups waited for.
        const bool all_ok = rec3::vote_all(ok, 5, NSTREAM * EPI_WG);
        if (all_ok) {
            float *red = reinterpret_cast<float *>(smem + L.red);  // [2 * 64 rows][64]
            const int rrow = sw * NBS_MAX + m;
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
                for (int u = 0; u < UPT; ++u)
                    red[rrow * 64 + g * UPC + uo + u] = valid ? dbacc[g][u] : 0.f;
            rec::named_bar(5, NSTREAM * EPI_WG);
            if (et < 64) {
                float sum = 0.f;
                for (int r = 0; r < NSTREAM * NBS_MAX; ++r) sum += red[r * 64 + et];
                const int g = et / UPC, u = et % UPC;  // g: the role
                const int blk = IJFO && (g == 1 || g == 2) ? 3 - g : g;
                float *dst = p.db_part + (long long)gi * G4 + (long long)blk * H + j0 +
                             (int)kpart * UPC + u;
                *dst = first ? sum : *dst + sum;  // launches of one call run in order
            }
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();
    if (warp == 2) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace rec4
}  // namespace lstm
