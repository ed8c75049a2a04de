// Recurrent kernels (16-bit operands: bf16, or fp16 for the page's FLOAT16
// data type; fp32 accumulation) with their weights resident in tensor memory: the
// tcgen05.mma A operand is read from TMEM, which leaves shared memory to the
// streamed operands and the cluster exchange.
//
// Forward (fwd3_kernel, "SingleLayerLstmGrad", forward-formula table, with the
// input concatenation of the operator page): the x-part of the gate
// pre-activation is contracted inside the recurrence instead of by a separate
// GEMM.  Per step the CTA accumulates W_x x_t (its K-slice of I) into the step's
// TMEM accumulator before the step's h_{t-1} arrives -- those MMAs depend on
// no other CTA, so they run while the tensor pipe would otherwise wait for the
// previous step's exchange and group barrier -- and then adds W_h h_{t-1}.  The
// work split, the DSMEM reduce-scatter and the epilogue are those of the
// cluster kernel in tc_recur2.cuh; the bias is added in the epilogue.
//
// Backward recurrence: "SingleLayerLstmGrad", backward pass, steps 1-6: per reverse time
// step, delta h = dG_{t+1} W_h (the K = 4H contraction) feeds the pointwise
// gradient of the cell, and the step's dG_t feeds the next contraction.
//
// Work split (same grid as the cluster kernel in tc_recur2.cuh): clusters of 8
// CTAs; a cluster owns 128 hidden units and one group of up to 128 batch rows;
// CTA k of the cluster contracts K-part k of the 4H axis (H/2 wide) and
// finalises 16 of the 128 units after a reduce-scatter over DSMEM.
//
// What differs from that kernel: the CTA's slice of W_h^T (128 units x H/2 of
// K, 128 KB of 16-bit values) is the MMA's A operand in TMEM (tcgen05.mma with A from
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

template <class E>  // E: the 16-bit compute type, __nv_bfloat16 or __half
struct Bwd3Params {
    CUtensorMap map_dg;               // dG [T*B][4H], box {64, NBr}
    const E *wt;                      // W_h^T [H][4H]
    const E *dy, *dhT, *gates;
    const float *dcT, *cells, *c0;
    E *dG;
    float *dh0, *dc0, *db_part;
    float *dc_carry;  // [B][H]: delta c between the launches of a chunked call
    // variable length (MASKED kernels): mask [T][B][H], 1 = real step,
    // 0 = padding; dhp_carry [B][H]: the delta h that padding passes to
    // h_{t-1}, between the launches of a chunked call
    const E *mask;
    float *dhp_carry;
    Ctrl *ctrl;
    int T, B, H, U, G, NBr, kcc, stages;
    int i0, i1;       // this launch runs epilogue iterations i0 .. i1-1 (step T-1-i)
    int reverse;      // direction "REDIRECTIONAL": recurrence step s is at time T-1-s
    int bar_base;     // first of the call's G step counters in ctrl->bar
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

// MASKED: variable-length mask; IJFO: gate_order "ijfo" (a template argument,
// not a runtime one: the epilogue is at the register limit of its launch)
template <class E, bool MASKED, bool IJFO>
__global__ void __launch_bounds__(THREADS, 1) bwd3_kernel(const __grid_constant__ Bwd3Params<E> p) {
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
    volatile int *cluster_bad = abort_flag + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int us = cid % p.U, gi = cid / p.U;
    const int j0 = us * UNITS, b0 = gi * p.NBr;
    const int H = p.H, B = p.B, T = p.T, kcc = p.kcc, NBr = p.NBr, stages = p.stages;
    // A call may run in several launches over consecutive ranges of reverse
    // time.  Epilogue iteration i >= 1 consumes MMA iteration i; the launch
    // that ends the call also runs MMA iteration T (delta h_0).
    const int i0 = p.i0, i1 = p.i1;
    const bool first = i0 == 0, last = i1 == T;
    const int mma_lo = i0 > 1 ? i0 : 1, mma_hi = last ? T : i1 - 1;
    // time of recurrence step s of the forward pass
    auto tau = [&](int s) { return p.reverse ? T - 1 - s : s; };
    const int kslice = kcc * 64;              // this CTA's part of the 4H axis
    const int kbase = (int)kpart * kslice;
    unsigned int *ctr = &p.ctrl->bar[p.bar_base + gi];
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
        *cluster_bad = tc::cluster_nctarank() != (uint32_t)KS;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*cluster_bad) {  // a launch without the cluster shape: report, touch no peer
        if (threadIdx.x == 0) atomicCAS(&p.ctrl->status, 0u, 2u);  // LSTM_ERR_UNSUPPORTED
        if (warp == 1) {
            tc::tc_fence_after();
            tc::tmem_dealloc(*tmem_slot, TMEM_COLS);
        }
        return;
    }
    tc::cluster_sync_all();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t a_bytes = (uint32_t)NBr * 128;  // rows loaded per chunk (NBr % 16 == 0)

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, ph = 0;
            bool aborted = false;
            // MMA iteration i consumes dG_{T-i}, written in iteration i-1
            for (int i = mma_lo; i <= mma_hi && !aborted; ++i) {
                if (!rec::wait_counter(ctr, group_ctas * (unsigned)i, p.ctrl, abort_flag, 0x601,
                                       p.wait_ns)) {
                    aborted = true;
                    break;
                }
                // acquire above, then the proxy fence: the TMA reads below see
                // every dG store the group released
                tc::fence_proxy_async_global();
                const int row0 = tau(T - i) * B + b0;  // dG of step T-i
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
            const uint32_t idesc = tc::idesc_f16kind_f32(Elem<E>::kFmt, UNITS, NBr, 0, 0);
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
            for (int i = mma_lo; ok && i <= mma_hi; ++i) {
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
            // TMEM lanes 32q + lane, two elements per column (lower K in the low half)
            const int u = 32 * q + lane;
            const E *src =
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
        // row block of each gate role i, f, g, o (gate_order); the registers
        // below hold the gates by role
        constexpr int kBlk[4] = {0, IJFO ? 2 : 1, IJFO ? 1 : 2, 3};
        uint4 gpk[4], dypk;  // prefetched gates and dy of the next step, still packed bf16
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
                for (int s = 0; s < 4; ++s) {
                    uint32_t v[16];
                    tc::tmem_ld16(tmem_base + ((uint32_t)(32 * q) << 16) + D_COL +
                                      (uint32_t)(hh * 64 + 16 * s),
                                  v);
                    tc::tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int n = hh * 64 + 16 * s + 4 * k;
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
                    // (__fmul_rn: no contraction into the sums below, so that
                    // m = 1 rounds exactly as the unmasked kernel does)
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
                }
                if (valid) {
                    float ri[UPT], rf[UPT], rg[UPT], ro[UPT];  // db sums the stored values
                    x8_to_f32<E>(vi, ri);
                    x8_to_f32<E>(vf, rf);
                    x8_to_f32<E>(vg, rg);
                    x8_to_f32<E>(vo, ro);
#pragma unroll
                    for (int u = 0; u < UPT; ++u) {
                        dbacc[0][u] += ri[u];
                        dbacc[1][u] += rf[u];
                        dbacc[2][u] += rg[u];
                        dbacc[3][u] += ro[u];
                    }
                }
            }
            rec::named_bar(1, EPI_THREADS);
            if (et == 0) {
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
            ok = ok && read_dh(dh0v);  // uniform over the epilogue threads
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
                const int g = et / UPC, u = et % UPC;  // g: the role
                const int blk = IJFO && (g == 1 || g == 2) ? 3 - g : g;
                float *dst = p.db_part + (long long)gi * G4 + (long long)blk * H + j0 + (int)kpart * UPC + u;
                *dst = first ? sum : *dst + sum;  // launches of one call run in order
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

// =========================================================================
// forward with the input projection fused
// =========================================================================
constexpr int F3_MAXC = 16;         // K chunks (of 64) per operand ring
constexpr int F3_BAR_BYTES = 1024;

template <class E>  // E: the 16-bit compute type, __nv_bfloat16 or __half
struct Fwd3Params {
    CUtensorMap map_y;                // y  [T*B][H], box {64, NB}: h_{t-1}
    CUtensorMap map_h0;               // h0 [B][H],   box {64, NB}
    CUtensorMap map_x;                // x  [T*B][I], box {64, NB}
    const E *W;                       // [4H][H + I]: W_h | W_x
    const E *bias;                    // [4H] or NULL
    const float *c0;
    // variable length (MASKED kernels): mask [T][B][H], 1 = real step,
    // 0 = padding (which keeps h_{t-1}, c_{t-1}); h0 [B][H] or NULL
    const E *mask, *h0;
    int reverse;  // direction "REDIRECTIONAL": recurrence step s is at time T-1-s
    int ijfo;     // gate_order "ijfo": row blocks i, j (= g), f, o instead of i, f, j, o
    E *y, *gates, *hT;
    float *cells, *cT;
    Ctrl *ctrl;
    int T, B, H, I, R, G, kcc, kcx, has_h0;
    int bar_base;  // first of this launch's G * SPLIT step counters in ctrl->bar
    int fault_skip_cta;
    unsigned long long wait_ns;
};

// TMEM columns: two accumulators of NB, then the W_h slice (kcc x 32), then the
// W_x slice (kcx x 32)
__host__ __device__ constexpr int fwd3_tmem_cols(int NB, int kcc, int kcx) {
    return 2 * NB + 32 * (kcc + kcx);
}

// ring_h: kcc chunks of h_{t-1} (NB rows x 64 K); ring_x: kcx chunks of x_t;
// recv / xbuf / send as in the cluster forward kernel.  One batch stream
// (SPLIT = 1): send aliases ring_h, idle between a step's last MMA and the
// next step's h loads, when it is large enough.  Two interleaved streams
// (SPLIT = 2): one stream's h loads and MMAs overlap the other's exchange, so
// send has a place of its own, and recv, xbuf and send are one per stream.
struct Fwd3Smem {
    int ring_h, ring_x, recv, xbuf, send, bars, total;
    __host__ __device__ Fwd3Smem(int kcc, int kcx, int NB, int KS, int SPLIT = 1) {
        const int NBc = NB / KS;
        const int hbytes = kcc * NB * 128, xbytes = kcx * NB * 128;
        const int part_bytes = (KS - 1) * NBc * rec2::F_ROWS * 4;
        const int xbuf_bytes = 4 * NBc * rec2::F_UNITS * 4;
        ring_h = 0;
        ring_x = hbytes;
        recv = ring_x + xbytes;
        if (SPLIT == 1) {
            xbuf = recv + part_bytes;
            send = hbytes >= part_bytes ? ring_h : xbuf + xbuf_bytes;
            bars = send == ring_h ? xbuf + xbuf_bytes : send + part_bytes;
        } else {
            xbuf = recv + 2 * part_bytes;  // one gate-exchange block per stream
            send = xbuf + 2 * xbuf_bytes;
            bars = send + 2 * part_bytes;
        }
        bars = (bars + 15) & ~15;
        total = bars + F3_BAR_BYTES;
    }
};

// AND of `v` over the `n` threads that use named barrier `id`
__device__ __forceinline__ bool vote_all(bool v, int id, int n) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// SPLIT = 2: the cluster's batch group of 2 NB rows is two independent
// streams of NB rows, processed in alternating virtual steps v = 2t + half
// (each with its own group barrier), so that one stream's h-part MMAs run
// while the other's partial sums cross DSMEM.  NB is the batch width of one
// virtual step, and each stream has an epilogue warpgroup of its own, so that
// the two streams' epilogues also overlap each other.
template <class E, int NB, int KS, bool MASKED, int SPLIT = 1>
__global__ void __launch_bounds__(rec2::F_THREADS, 1) fwd3_kernel(const __grid_constant__ Fwd3Params<E> p) {
    using rec2::F_ROWS;
    using rec2::F_UNITS;
    using rec2::F_EPI_THREADS;
    constexpr int NBc = NB / KS;       // batch columns finalised by this CTA
    constexpr int NBh = NBc / 2;       // columns each of the two warps of a quarter moves
    constexpr int NP = (NBc + 7) / 8;  // (unit, batch) pairs per epilogue thread
    constexpr int VW = NBh >= 4 ? 4 : 2;  // floats per staged vector / receive chunk
    static_assert(NBc >= 4 && NBc % 4 == 0 && NBc <= 32, "columns per CTA");
    static_assert(SPLIT == 1 || SPLIT == 2, "one or two batch streams");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int kcc = p.kcc, kcx = p.kcx;
    const Fwd3Smem L(kcc, kcx, NB, KS, SPLIT);
    uint8_t *ring_h = smem + L.ring_h;
    uint8_t *ring_x = smem + L.ring_x;
    // recv / send: [SPLIT buffers][KS-1 partners][NBc/VW chunks][128 rows][VW]
    float *recv = (float *)(smem + L.recv);
    float *xbuf = (float *)(smem + L.xbuf);  // [4 gates][NBc][32 units]
    float *send = (float *)(smem + L.send);
    uint64_t *bars = (uint64_t *)(smem + L.bars);
    uint64_t *h_full = bars;
    uint64_t *h_empty = bars + F3_MAXC;
    uint64_t *x_full = bars + 2 * F3_MAXC;
    uint64_t *x_empty = bars + 3 * F3_MAXC;
    uint64_t *w_ready = bars + 4 * F3_MAXC;  // W_h and W_x slices written to TMEM
    uint64_t *mma_done = w_ready + 1;        // [2]: accumulator complete
    uint64_t *d_free = w_ready + 3;          // [2]: accumulator read out by the epilogue
    uint64_t *recv_full = w_ready + 5;       // [SPLIT]
    uint32_t *tmem_slot = (uint32_t *)(w_ready + 7);
    volatile int *abort_flag = (volatile int *)(w_ready + 8);
    volatile int *cluster_bad = abort_flag + 1;

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const uint32_t kpart = tc::cluster_rank();
    const int cid = blockIdx.x / KS;
    const int rs = cid % p.R, gi = cid / p.R;
    const int u0 = rs * F_UNITS, b0 = gi * NB * SPLIT;  // the group's first batch row
    const int H = p.H, B = p.B, T = p.T, I = p.I;
    const int kbase = (int)kpart * kcc * 64;  // this CTA's K range of W_h / h
    const int xbase = (int)kpart * kcx * 64;  // and of W_x / x
    // time of recurrence step s (step s reads the state step s-1 left)
    auto tau = [&](int s) { return p.reverse ? T - 1 - s : s; };
    const uint32_t WH_COL = 2 * NB, WX_COL = 2 * NB + 32 * kcc;
    unsigned int *ctr = &p.ctrl->bar[p.bar_base + gi * SPLIT];  // + stream: one per stream
    const int V = T * SPLIT;                        // virtual steps
    const unsigned int group_ctas = (unsigned)(p.R * KS);
    constexpr uint32_t TMEM_COLS = 512;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kcc; ++i) {
            tc::mbar_init(&h_full[i], 1);
            tc::mbar_init(&h_empty[i], 1);
        }
        for (int i = 0; i < kcx; ++i) {
            tc::mbar_init(&x_full[i], 1);
            tc::mbar_init(&x_empty[i], 1);
        }
        tc::mbar_init(w_ready, F_EPI_THREADS);
        tc::mbar_init(&mma_done[0], 1);
        tc::mbar_init(&mma_done[1], 1);
        tc::mbar_init(&d_free[0], 1);
        tc::mbar_init(&d_free[1], 1);
        // one local arrival (with the expected bytes) per (virtual) step
        for (int i = 0; i < SPLIT; ++i) tc::mbar_init(&recv_full[i], 1);
        *abort_flag = 0;
        *cluster_bad = tc::cluster_nctarank() != (uint32_t)KS;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::tc_fence_before();
    __syncthreads();
    if (*cluster_bad) {  // a launch without the cluster shape: report, touch no peer
        if (threadIdx.x == 0) atomicCAS(&p.ctrl->status, 0u, 2u);  // LSTM_ERR_UNSUPPORTED
        if (warp == 1) {
            tc::tc_fence_after();
            tc::tmem_dealloc(*tmem_slot, TMEM_COLS);
        }
        return;
    }
    tc::cluster_sync_all();  // every CTA's barriers exist before any remote arrival
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            constexpr uint32_t CHUNK = NB * 128;
            // loads issued per chunk, so that an aborted CTA can let them land
            int rounds_h = 0, part_h = 0, rounds_x = 0, part_x = 0;
            uint32_t phh = 0, phx = 0;
            bool aborted = false;
            auto load_x = [&](int v) -> bool {  // x rows of virtual step v
                const int row = tau(v / SPLIT) * B + b0 + (v % SPLIT) * NB;
                for (int c = 0; c < kcx; ++c) {
                    if (!tc::mbar_wait(&x_empty[c], phx ^ 1, p.ctrl, abort_flag, 0x702, p.wait_ns))
                        return false;
                    tc::mbar_arrive_expect_tx(&x_full[c], CHUNK);
                    tc::tma_load_2d(ring_x + c * CHUNK, &p.map_x, &x_full[c], xbase + 64 * c, row);
                    part_x = c + 1;
                }
                phx ^= 1;
                ++rounds_x;
                part_x = 0;
                return true;
            };
            aborted = !load_x(0);
            for (int v = 0; v < V && !aborted; ++v) {
                const int t = v / SPLIT, bh = b0 + (v % SPLIT) * NB;  // step, first row
                if (t > 0) {
                    if (!rec::wait_counter(ctr + v % SPLIT, group_ctas * (unsigned)t, p.ctrl,
                                           abort_flag, 0x701, p.wait_ns)) {
                        aborted = true;
                        break;
                    }
                    // the group's generic-proxy stores were released to this
                    // thread's acquire; order the TMA (async-proxy) reads after it
                    tc::fence_proxy_async_global();
                }
                if (t > 0 || p.has_h0) {
                    const CUtensorMap *m = t > 0 ? &p.map_y : &p.map_h0;
                    const int row0 = t > 0 ? tau(t - 1) * B + bh : bh;
                    for (int c = 0; c < kcc && !aborted; ++c) {
                        if (!tc::mbar_wait(&h_empty[c], phh ^ 1, p.ctrl, abort_flag, 0x703,
                                           p.wait_ns)) {
                            aborted = true;
                            break;
                        }
                        tc::mbar_arrive_expect_tx(&h_full[c], CHUNK);
                        tc::tma_load_2d(ring_h + c * CHUNK, m, &h_full[c], kbase + 64 * c, row0);
                        part_h = c + 1;
                    }
                    if (aborted) break;
                    phh ^= 1;
                    ++rounds_h;
                    part_h = 0;
                }
                // the next virtual step's x does not depend on the group: issue it now
                if (v + 1 < V && !load_x(v + 1)) aborted = true;
            }
            if (aborted) {  // let every issued copy land before the CTA can exit
                for (int c = 0; c < kcc; ++c) {
                    const int n = rounds_h + (c < part_h ? 1 : 0);
                    if (n > 0) tc::mbar_wait(&h_full[c], (uint32_t)((n - 1) & 1), nullptr, nullptr, 0, 200000000ull);
                }
                for (int c = 0; c < kcx; ++c) {
                    const int n = rounds_x + (c < part_x ? 1 : 0);
                    if (n > 0) tc::mbar_wait(&x_full[c], (uint32_t)((n - 1) & 1), nullptr, nullptr, 0, 200000000ull);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // D[128 gate rows][NB] = W_x slice (TMEM) x x_t chunk^T (+)
            //                        W_h slice (TMEM) x h_{t-1} chunk^T
            const uint32_t idesc = tc::idesc_f16kind_f32(Elem<E>::kFmt, F_ROWS, NB, 0, 0);
            const uint64_t hi = tc::smem_desc_sw128(0, 16, 1024);
            const uint64_t rh_lo0 = tc::smem_u32(ring_h) >> 4, rx_lo0 = tc::smem_u32(ring_x) >> 4;
            constexpr uint32_t CSTEP = (NB * 128) >> 4;
            uint32_t phh = 0, phx = 0;
            bool ok = tc::mbar_wait(w_ready, 0, p.ctrl, abort_flag, 0x704, p.wait_ns);
            tc::tc_fence_after();
            // x-part of step s into accumulator s & 1, once the epilogue has
            // read that accumulator's previous use (step s - 2)
            auto x_part = [&](int s) -> bool {
                const int acc = s & 1;
                if (!tc::mbar_wait(&d_free[acc], (uint32_t)(((s >> 1) & 1) ^ 1), p.ctrl, abort_flag,
                                   0x705, p.wait_ns))
                    return false;
                tc::tc_fence_after();
                const uint32_t d = tmem_base + acc * NB;
                for (int c = 0; c < kcx; ++c) {
                    if (!tc::mbar_wait(&x_full[c], phx, p.ctrl, abort_flag, 0x706, p.wait_ns))
                        return false;
                    tc::tc_fence_after();
                    const uint64_t bd = hi | (rx_lo0 + c * CSTEP);
                    const uint32_t a = tmem_base + WX_COL + 32 * c;
                    tc::mma_bf16_ts(d, a, bd, idesc, c != 0);
                    tc::mma_bf16_ts(d, a + 8, bd + 2, idesc, 1);
                    tc::mma_bf16_ts(d, a + 16, bd + 4, idesc, 1);
                    tc::mma_bf16_ts(d, a + 24, bd + 6, idesc, 1);
                    tc::mma_commit(&x_empty[c]);
                }
                phx ^= 1;
                return true;
            };
            ok = ok && x_part(0);
            for (int v = 0; ok && v < V; ++v) {
                const int acc = v & 1;
                const uint32_t d = tmem_base + acc * NB;
                if (v >= SPLIT || p.has_h0) {  // h_{t-1} is zero at t = 0 without h0
                    for (int c = 0; c < kcc; ++c) {
                        if (!tc::mbar_wait(&h_full[c], phh, p.ctrl, abort_flag, 0x707, p.wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                        const uint64_t bd = hi | (rh_lo0 + c * CSTEP);
                        const uint32_t a = tmem_base + WH_COL + 32 * c;
                        tc::mma_bf16_ts(d, a, bd, idesc, 1);
                        tc::mma_bf16_ts(d, a + 8, bd + 2, idesc, 1);
                        tc::mma_bf16_ts(d, a + 16, bd + 4, idesc, 1);
                        tc::mma_bf16_ts(d, a + 24, bd + 6, idesc, 1);
                        tc::mma_commit(&h_empty[c]);
                    }
                    if (!ok) break;
                    phh ^= 1;
                }
                tc::mma_commit(&mma_done[acc]);
                if (v + 1 < V) ok = x_part(v + 1);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;  // 0..255
        const int q = warp & 3;           // TMEM lane quarter = gate of the row read
        const int hh = (warp - 2) >> 2;   // which half of each column block it moves
        const int mrow = 32 * q + lane;   // row of the partial tile: gate q, unit lane
        {
            // W rows q*H + u0 + lane: this warp's half of the CTA's K range of
            // W_h and of W_x (zero past I) -> TMEM lane mrow, two elements per column
            const E *wrow = p.W + (long long)(q * H + u0 + lane) * (H + I);
            const uint32_t trow = tmem_base + ((uint32_t)(32 * q) << 16);
            const int hn = kcc * 2;  // 16-element groups per half of the W_h range
            for (int n = 0; n < hn; ++n) {
                const E *src = wrow + kbase + hh * kcc * 32 + 16 * n;
                const uint4 x0 = __ldg(reinterpret_cast<const uint4 *>(src));
                const uint4 x1 = __ldg(reinterpret_cast<const uint4 *>(src + 8));
                const uint32_t r[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                tc::tmem_st8(trow + WH_COL + (uint32_t)(hh * kcc * 16 + 8 * n), r);
            }
            const int xn = kcx * 2;
            for (int n = 0; n < xn; ++n) {
                const int e = xbase + hh * kcx * 32 + 16 * n;  // first x feature of the group
                const E *src = wrow + H + e;
                const uint4 z = make_uint4(0, 0, 0, 0);
                const uint4 x0 = e < I ? __ldg(reinterpret_cast<const uint4 *>(src)) : z;
                const uint4 x1 = e + 8 < I ? __ldg(reinterpret_cast<const uint4 *>(src + 8)) : z;
                const uint32_t r[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                tc::tmem_st8(trow + WX_COL + (uint32_t)(hh * kcx * 16 + 8 * n), r);
            }
            tc::tmem_st_wait();
            tc::tc_fence_before();
            tc::mbar_arrive(w_ready);
        }
        // first batch row finalised here in virtual steps of stream `half`
        auto col0 = [&](int half) { return b0 + half * NB + (int)kpart * NBc; };
        constexpr uint32_t PART_BYTES = NBc * F_ROWS * 4;  // one partner's partial tile
        constexpr int BUF_FLOATS = (KS - 1) * (int)PART_BYTES / 4;  // one recv / send buffer
        // position of destination d among this CTA's partners (its send block),
        // and of this CTA among d's sources (its receive slot at d)
        auto dst_pos = [&](int d) { return d < (int)kpart ? d : d - 1; };
        auto src_slot = [&](int d) { return (int)kpart < d ? (int)kpart : (int)kpart - 1; };
        if constexpr (SPLIT == 2) {
            // One epilogue warpgroup per stream (warps 2-5: stream 0, 6-9:
            // stream 1), each with one warp per TMEM lane quarter, its own
            // named barriers, receive / staging / gate-exchange blocks and
            // state: while one stream waits for its partials or its group
            // barrier, the other's read-out and pointwise work proceed.
            constexpr int WG = F_EPI_THREADS / 2;
            constexpr int NP2 = NBc * F_UNITS / WG;  // (unit, column) pairs per thread
            static_assert(NBc * F_UNITS % WG == 0, "pairs per warpgroup thread");
            const int sw = hh, wt = et - sw * WG;  // stream, thread within the warpgroup
            const int bar_sync = 1 + 2 * sw, bar_vote = 2 + 2 * sw;
            const int bc0 = col0(sw);
            float *rv = recv + sw * BUF_FLOATS, *sd = send + sw * BUF_FLOATS;
            float *xb = xbuf + sw * (4 * NBc * F_UNITS);  // [4 gates][NBc][32 units]
            uint64_t *rf = &recv_full[sw];
            float c[NP2], hprev[NP2], mk[NP2], bias[4][NP2];
            auto pair_unit = [&](int k) { return (wt + WG * k) & 31; };
            auto pair_col = [&](int k) { return (wt + WG * k) >> 5; };
#pragma unroll
            for (int k = 0; k < NP2; ++k) {
                const int n = pair_col(k), b = bc0 + n, j = u0 + pair_unit(k);
                const bool v = b < B;
                c[k] = (p.c0 && v) ? p.c0[(long long)b * H + j] : 0.f;
                hprev[k] = (MASKED && p.h0 && v) ? to_f(p.h0[(long long)b * H + j]) : 0.f;
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    bias[g][k] = p.bias ? to_f(p.bias[g * H + j]) : 0.f;
            }
            auto load_mask = [&](int t) {  // this stream's mask of step t (time tau(t))
                const int tt = tau(t);
#pragma unroll
                for (int k = 0; k < NP2; ++k) {
                    const int b = bc0 + pair_col(k), j = u0 + pair_unit(k);
                    mk[k] = b < B ? to_f(p.mask[((long long)tt * B + b) * H + j]) : 0.f;
                }
            };
            if (MASKED) load_mask(0);
            uint32_t dph = 0, rph = 0;
            for (int t = 0; t < T; ++t) {
                const bool w = tc::mbar_wait(&mma_done[sw], dph, p.ctrl, abort_flag, 0x708,
                                             p.wait_ns);
                if (!vote_all(w, bar_vote, WG)) break;
                dph ^= 1;
                tc::tc_fence_after();
                float own[NBc];
#pragma unroll
                for (int d = 0; d < KS; ++d) {
#pragma unroll
                    for (int h2 = 0; h2 < 2; ++h2) {
                        uint32_t tv[NBh];
                        rec2::tmem_ld_cols<NBh>(tmem_base + ((uint32_t)(32 * q) << 16) + sw * NB +
                                                    d * NBc + h2 * NBh,
                                                tv);
                        tc::tmem_ld_wait();
                        if (d == (int)kpart) {
#pragma unroll
                            for (int n = 0; n < NBh; ++n) own[h2 * NBh + n] = __uint_as_float(tv[n]);
                        } else {
                            float *blk = sd + dst_pos(d) * (PART_BYTES / 4);
#pragma unroll
                            for (int k = 0; k < NBh / VW; ++k) {
                                const int ch = h2 * (NBh / VW) + k;
                                float *a = blk + (ch * F_ROWS + mrow) * VW;
                                if constexpr (VW == 4)
                                    *reinterpret_cast<float4 *>(a) = make_float4(
                                        __uint_as_float(tv[4 * k]), __uint_as_float(tv[4 * k + 1]),
                                        __uint_as_float(tv[4 * k + 2]), __uint_as_float(tv[4 * k + 3]));
                                else
                                    *reinterpret_cast<float2 *>(a) = make_float2(
                                        __uint_as_float(tv[2 * k]), __uint_as_float(tv[2 * k + 1]));
                            }
                        }
                    }
                }
                tc::tc_fence_before();
                if (KS > 1) tc::fence_proxy_async_smem();  // staged partials -> bulk copies
                rec::named_bar(bar_sync, WG);
                // accumulator read out: the MMA thread may start this stream's next x-part in it
                if (wt == 0) tc::mbar_arrive(&d_free[sw]);
                if (KS > 1) {
                    if (wt == 0) {
                        tc::mbar_arrive_expect_tx(rf, (KS - 1) * PART_BYTES);
                        const uint32_t recv_lo = tc::smem_u32(rv), bar_lo = tc::smem_u32(rf);
#pragma unroll
                        for (int s = 1; s < KS; ++s) {
                            const int d = ((int)kpart + s) % KS;
                            tc::bulk_copy_to_peer(
                                tc::map_rank(recv_lo + (uint32_t)src_slot(d) * PART_BYTES, (uint32_t)d),
                                sd + dst_pos(d) * (PART_BYTES / 4), PART_BYTES,
                                tc::map_rank(bar_lo, (uint32_t)d));
                        }
                        tc::bulk_commit();
                    }
                    const bool w2 = tc::mbar_wait_cluster(rf, rph, p.ctrl, abort_flag, 0x709,
                                                          p.wait_ns);
                    if (!vote_all(w2, bar_vote, WG)) break;
                    rph ^= 1;
#pragma unroll
                    for (int sl = 0; sl < KS - 1; ++sl) {
                        const float *src = rv + sl * F_ROWS * NBc;
#pragma unroll
                        for (int ch = 0; ch < NBc / VW; ++ch) {
                            const float *a = src + (ch * F_ROWS + mrow) * VW;
                            if constexpr (VW == 4) {
                                const float4 x = *reinterpret_cast<const float4 *>(a);
                                own[4 * ch] += x.x;
                                own[4 * ch + 1] += x.y;
                                own[4 * ch + 2] += x.z;
                                own[4 * ch + 3] += x.w;
                            } else {
                                const float2 x = *reinterpret_cast<const float2 *>(a);
                                own[2 * ch] += x.x;
                                own[2 * ch + 1] += x.y;
                            }
                        }
                    }
                }
#pragma unroll
                for (int n = 0; n < NBc; ++n) xb[(q * NBc + n) * F_UNITS + lane] = own[n];
                rec::named_bar(bar_sync, WG);
                const int tt = tau(t);  // time of this step
                const int fb = p.ijfo ? 2 : 1, gb = 3 - fb;  // forget / candidate row blocks
                E *yt = p.y + (long long)tt * B * H;
                E *gt = p.gates + (long long)tt * B * 4 * H;
                float *ct = p.cells + (long long)tt * B * H;
                float gsave[4][NP2];
#pragma unroll
                for (int k = 0; k < NP2; ++k) {
                    const int n = pair_col(k), uu = pair_unit(k);
                    const int b = bc0 + n, j = u0 + uu;
                    const float bf_ = fb == 1 ? bias[1][k] : bias[2][k];
                    const float bg_ = fb == 1 ? bias[2][k] : bias[1][k];
                    const float ig = rec::sigmoid_fast(xb[(0 * NBc + n) * F_UNITS + uu] + bias[0][k]);
                    const float fg = rec::sigmoid_fast(xb[(fb * NBc + n) * F_UNITS + uu] + bf_);
                    const float gg = rec::tanh_fast(xb[(gb * NBc + n) * F_UNITS + uu] + bg_);
                    const float og = rec::sigmoid_fast(xb[(3 * NBc + n) * F_UNITS + uu] + bias[3][k]);
                    const float cn = fg * c[k] + ig * gg;
                    float h = og * rec::tanh_fast(cn);
                    if (MASKED) {  // padding keeps the previous state
                        c[k] = mk[k] * cn + (1.f - mk[k]) * c[k];
                        h = mk[k] * h + (1.f - mk[k]) * hprev[k];
                        hprev[k] = h;
                    } else {
                        c[k] = cn;
                    }
                    gsave[0][k] = ig; gsave[1][k] = fg; gsave[2][k] = gg; gsave[3][k] = og;
                    if (b < B) {
                        const long long o = (long long)b * H + j;
                        yt[o] = from_f<E>(h);  // h_t: what the other CTAs wait for
                        if (t == T - 1) {
                            p.hT[o] = from_f<E>(h);
                            p.cT[o] = c[k];
                        }
                    }
                }
                // this step's copies must have read the staging block before
                // the next step stages into it
                if (KS > 1 && wt == 0) tc::bulk_wait_read_all();
                rec::named_bar(bar_sync, WG);  // y[t] stored; xb and rv free again
                if (wt == 0 && (int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr + sw, 1u);
                // saved state for the backward pass, outside the writes the
                // arrival's release has to cover
#pragma unroll
                for (int k = 0; k < NP2; ++k) {
                    const int n = pair_col(k), uu = pair_unit(k);
                    const int b = bc0 + n, j = u0 + uu;
                    if (b >= B) continue;
                    ct[(long long)b * H + j] = c[k];
                    E *g4 = gt + (long long)b * 4 * H + j;
                    g4[0] = from_f<E>(gsave[0][k]);
                    g4[fb * H] = from_f<E>(gsave[1][k]);
                    g4[gb * H] = from_f<E>(gsave[2][k]);
                    g4[3 * H] = from_f<E>(gsave[3][k]);
                }
                if (MASKED && t + 1 < T) load_mask(t + 1);
            }
            if (wt == 0) tc::bulk_wait_all();  // no copy of this CTA still in flight at exit
        } else {
            const int bc0 = col0(0);  // first batch row finalised here
            // pointwise pairs of this thread: pair index et + 256 k -> unit, column
            float c[NP], bias[4][NP];
            float hprev[NP], mk[NP];  // MASKED: h_{t-1} of each pair, and step t's mask
            auto pair_unit = [&](int k) { return (et + F_EPI_THREADS * k) & 31; };
            auto pair_col = [&](int k) { return (et + F_EPI_THREADS * k) >> 5; };
    #pragma unroll
            for (int k = 0; k < NP; ++k) {
                const int n = pair_col(k), b = bc0 + n, j = u0 + pair_unit(k);
                const bool v = n < NBc && b < B;
                c[k] = (p.c0 && v) ? p.c0[(long long)b * H + j] : 0.f;
                if (MASKED) hprev[k] = (p.h0 && v) ? to_f(p.h0[(long long)b * H + j]) : 0.f;
    #pragma unroll
                for (int g = 0; g < 4; ++g)
                    bias[g][k] = p.bias ? to_f(p.bias[g * H + j]) : 0.f;
            }
            auto load_mask = [&](int s) {  // mask of step s (time tau(s))
                const int t = tau(s);
    #pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const int n = pair_col(k), b = bc0 + n, j = u0 + pair_unit(k);
                    mk[k] = (n < NBc && b < B)
                                ? to_f(p.mask[((long long)t * B + b) * H + j]) : 0.f;
                }
            };
            if (MASKED) load_mask(0);
            uint32_t dph[2] = {0, 0}, rph = 0;
            for (int t = 0; t < T; ++t) {
                const int acc = t & 1;
                const bool w = tc::mbar_wait(&mma_done[acc], dph[acc], p.ctrl, abort_flag, 0x708,
                                             p.wait_ns);
                if (!rec::epi_vote_all_n<F_EPI_THREADS>(w)) break;
                dph[acc] ^= 1;
                tc::tc_fence_after();
                float own[NBh];
    #pragma unroll
                for (int d = 0; d < KS; ++d) {
                    uint32_t v[NBh];
                    rec2::tmem_ld_cols<NBh>(
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
                if (KS > 1) tc::fence_proxy_async_smem();  // staged partials -> bulk copies
                rec::named_bar(1, F_EPI_THREADS);
                // accumulator read out: the MMA thread may start step t + 2's x-part in it
                if (et == 0) tc::mbar_arrive(&d_free[acc]);
                if (KS > 1) {
                    if (et == 0) {
                        tc::mbar_arrive_expect_tx(recv_full, (KS - 1) * PART_BYTES);
                        const uint32_t recv_lo = tc::smem_u32(recv), bar_lo = tc::smem_u32(recv_full);
                        // rank kpart + s first: each CTA receives from one sender at a time
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
                    const bool w2 = tc::mbar_wait_cluster(recv_full, rph, p.ctrl, abort_flag, 0x709,
                                                          p.wait_ns);
                    if (!rec::epi_vote_all_n<F_EPI_THREADS>(w2)) break;
                    rph ^= 1;
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
                }
    #pragma unroll
                for (int n = 0; n < NBh; ++n) xbuf[(q * NBc + hh * NBh + n) * F_UNITS + lane] = own[n];
                rec::named_bar(1, F_EPI_THREADS);
                const int tt = tau(t);  // time of this step
                // row blocks of the forget gate and the candidate (gate_order)
                const int fb = p.ijfo ? 2 : 1, gb = 3 - fb;
                E *yt = p.y + (long long)tt * B * H;
                E *gt = p.gates + (long long)tt * B * 4 * H;
                float *ct = p.cells + (long long)tt * B * H;
                float gsave[4][NP];
    #pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const int n = pair_col(k), uu = pair_unit(k);
                    if (n >= NBc) continue;
                    const int b = bc0 + n, j = u0 + uu;
                    const float bf_ = fb == 1 ? bias[1][k] : bias[2][k];
                    const float bg_ = fb == 1 ? bias[2][k] : bias[1][k];
                    const float ig = rec::sigmoid_fast(xbuf[(0 * NBc + n) * F_UNITS + uu] + bias[0][k]);
                    const float fg = rec::sigmoid_fast(xbuf[(fb * NBc + n) * F_UNITS + uu] + bf_);
                    const float gg = rec::tanh_fast(xbuf[(gb * NBc + n) * F_UNITS + uu] + bg_);
                    const float og = rec::sigmoid_fast(xbuf[(3 * NBc + n) * F_UNITS + uu] + bias[3][k]);
                    const float cn = fg * c[k] + ig * gg;
                    float h = og * rec::tanh_fast(cn);
                    if (MASKED) {  // padding keeps the previous state
                        c[k] = mk[k] * cn + (1.f - mk[k]) * c[k];
                        h = mk[k] * h + (1.f - mk[k]) * hprev[k];
                        hprev[k] = h;
                    } else {
                        c[k] = cn;
                    }
                    gsave[0][k] = ig; gsave[1][k] = fg; gsave[2][k] = gg; gsave[3][k] = og;
                    if (b < B) {
                        const long long o = (long long)b * H + j;
                        yt[o] = from_f<E>(h);  // h_t: what the other CTAs wait for
                        if (t == T - 1) {
                            p.hT[o] = from_f<E>(h);
                            p.cT[o] = c[k];
                        }
                    }
                }
                rec::named_bar(1, F_EPI_THREADS);  // y[t] stored; xbuf and recv free again
                if (et == 0) {
                    // the staging block must be read out before this CTA's arrival
                    // lets the next step's TMA refill ring_h
                    if (KS > 1) tc::bulk_wait_read_all();
                    if ((int)blockIdx.x != p.fault_skip_cta) rec::red_release_add(ctr, 1u);
                }
                // saved state for the backward pass, outside the writes the
                // arrival's release has to cover
    #pragma unroll
                for (int k = 0; k < NP; ++k) {
                    const int n = pair_col(k), uu = pair_unit(k);
                    const int b = bc0 + n, j = u0 + uu;
                    if (n >= NBc || b >= B) continue;
                    ct[(long long)b * H + j] = c[k];
                    E *g4 = gt + (long long)b * 4 * H + j;
                    const int fb = p.ijfo ? 2 : 1, gb = 3 - fb;
                    g4[0] = from_f<E>(gsave[0][k]);
                    g4[fb * H] = from_f<E>(gsave[1][k]);
                    g4[gb * H] = from_f<E>(gsave[2][k]);
                    g4[3 * H] = from_f<E>(gsave[3][k]);
                }
                if (MASKED && t + 1 < T) load_mask(t + 1);
            }
            if (et == 0) tc::bulk_wait_all();  // no copy of this CTA still in flight at exit
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    tc::cluster_sync_all();  // no partner may still be writing into this CTA's smem
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace rec3
}  // namespace lstm
