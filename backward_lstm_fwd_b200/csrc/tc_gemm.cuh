// tc_gemm.cuh -- persistent tcgen05 / TMA GEMM core for 16-bit operands (bf16
// or fp16, one type per launch) with fp32 accumulation in TMEM, used for the time-parallel contractions of the path:
//   input projection   Gx = X W_x^T + b        (A = X K-major, B = W_x K-major)
//   dW                 dG^T [h_prev | x]        (A = dG MN-major, B = y / x MN-major)
//   dx                 dG W_x                  (A = dG K-major, B = W_x MN-major)
//
// One launch walks a table of up to four problems (each with up to two K
// segments drawn from different tensor maps), one 128 x 256 output tile per
// step of a static persistent schedule (sched_tile).  Warp roles:
//   warp 0      one thread issues TMA loads into a 4-stage shared-memory ring;
//   warp 1      allocates TMEM and one thread issues tcgen05.mma (M=128,
//               N=256, K=16 per instruction) into one of two accumulators;
//   warps 2-5   epilogue: TMEM -> registers -> (+ bias) -> fp32 global stores
//               (32-byte vector stores where the output is aligned for them),
//               overlapping the next tile's MMAs through the second accumulator.
#pragma once

#include <cuda.h>

#include "tc_ptx.cuh"

namespace lstm {
namespace tcg {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
static_assert(BK == 64, "the MMA issuer unrolls four K=16 steps per stage");
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 192;
constexpr int TMEM_COLS = 2 * BN;             // two fp32 accumulators of BN columns
constexpr int MAX_MAPS = 6, MAX_PROB = 4;
constexpr int MN_BOX_BYTES = 64 * BK * 2;     // one 64 (MN) x 64 (K) box: 8 KB
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct Seg {
    int a_map, b_map;  // indices into Params::maps
    int a_k0, b_k0;    // K coordinate of the segment's first block in each map
    int nkb;           // number of BK-deep K blocks
};

struct Problem {
    int M, N;                  // output extent
    int a_mn_major, b_mn_major;
    int a_mn0, b_mn0;          // MN coordinate of output row / column 0 in the maps
    int nseg;
    Seg seg[2];
    float *out;                // out[m * ldo + out_col0 + n]
    long long ldo;
    int out_col0;
    int accumulate;            // out += product (otherwise out = product)
    const void *bias;          // added per column n (operand type), or NULL
    int tiles_n, tile_begin, tile_end;
};

struct Params {
    CUtensorMap maps[MAX_MAPS];
    Problem prob[MAX_PROB];
    int nprob, total_tiles;
    uint32_t fmt;              // operand format of every problem: 0 = fp16, 1 = bf16
    Ctrl *ctrl;
};

__device__ __forceinline__ int locate(const Params &p, int tile, int &mt, int &nt) {
    int pi = 0;
    while (pi + 1 < p.nprob && tile >= p.prob[pi].tile_end) ++pi;
    const int local = tile - p.prob[pi].tile_begin;
    mt = local / p.prob[pi].tiles_n;
    nt = local % p.prob[pi].tiles_n;
    return pi;
}

// The tile of this CTA's k-th step of the static schedule: rounds of
// gridDim.x consecutive tiles, the first in CTA order and every later one in
// reverse CTA order.  The queue holds its largest tiles first, so the CTAs
// that drew the larger first-round tiles draw the last, partial round's
// tiles last, if at all (the last dW / dx chunk of the bench backward: 138
// instead of 156 K blocks on the busiest CTA against 119 on average).  Every
// round but the last is full, so a CTA's first tile past the queue ends it.
__device__ __forceinline__ int sched_tile(int k) {
    return k * (int)gridDim.x + (k == 0 ? (int)blockIdx.x : (int)gridDim.x - 1 - (int)blockIdx.x);
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t base, int mn_major, int k16) {
    // K-major: rows of 128 B (64 bf16 of K), 8-row groups 1024 B apart; a
    //          K=16 step moves 32 B inside the 128-byte swizzle row.
    // MN-major: 64-element MN chunks one 8 KB box apart (leading offset),
    //          8-row K groups 1024 B apart; a K=16 step moves two groups.
    return mn_major ? tc::smem_desc_sw128(base + k16 * 2048, MN_BOX_BYTES, 1024)
                    : tc::smem_desc_sw128(base + k16 * 32, 16, 1024);
}

__global__ void __launch_bounds__(NUM_THREADS, 1) gemm_kernel(const __grid_constant__ Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * A_BYTES;
    uint64_t *full = (uint64_t *)(sB + STAGES * B_BYTES);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = (uint32_t *)(tempty + 2);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(&full[s], 1);
            tc::mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(&tfull[a], 1);
            tc::mbar_init(&tempty[a], 4);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, TMEM_COLS);
        tc::tmem_relinquish();
    }
    if (warp == 0 && lane == 0)
        for (int i = 0; i < MAX_MAPS; ++i) tc::tma_prefetch_desc(&p.maps[i]);
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t stage = 0, phase = 0;
            uint32_t issued_parity[STAGES];
            bool issued[STAGES];
            for (int s = 0; s < STAGES; ++s) issued[s] = false, issued_parity[s] = 0;
            bool ok = true;
            for (int k = 0, tile; ok && (tile = sched_tile(k)) < p.total_tiles; ++k) {
                int mt, nt;
                const Problem &P = p.prob[locate(p, tile, mt, nt)];
                const int m0 = P.a_mn0 + mt * BM, n0 = P.b_mn0 + nt * BN;
                for (int sg = 0; ok && sg < P.nseg; ++sg) {
                    const Seg &S = P.seg[sg];
                    for (int kb = 0; kb < S.nkb; ++kb) {
                        if (!tc::mbar_wait(&empty[stage], phase ^ 1, p.ctrl, abort_flag, 0x101)) {
                            ok = false;
                            break;
                        }
                        tc::mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                        uint8_t *a = sA + stage * A_BYTES;
                        uint8_t *b = sB + stage * B_BYTES;
                        const CUtensorMap *am = &p.maps[S.a_map];
                        const CUtensorMap *bm = &p.maps[S.b_map];
                        const int ka = S.a_k0 + kb * BK, kbb = S.b_k0 + kb * BK;
                        if (!P.a_mn_major) {
                            tc::tma_load_2d(a, am, &full[stage], ka, m0);
                        } else {
#pragma unroll
                            for (int c = 0; c < BM / 64; ++c)
                                tc::tma_load_2d(a + c * MN_BOX_BYTES, am, &full[stage], m0 + 64 * c, ka);
                        }
                        if (!P.b_mn_major) {
                            tc::tma_load_2d(b, bm, &full[stage], kbb, n0);
                        } else {
#pragma unroll
                            for (int c = 0; c < BN / 64; ++c)
                                tc::tma_load_2d(b + c * MN_BOX_BYTES, bm, &full[stage], n0 + 64 * c, kbb);
                        }
                        issued[stage] = true;
                        issued_parity[stage] = phase;
                        if (++stage == STAGES) stage = 0, phase ^= 1;
                    }
                }
            }
            if (!ok) {
                // drain: let every copy this thread issued land before exiting
                for (int s = 0; s < STAGES; ++s)
                    if (issued[s])
                        tc::mbar_wait(&full[s], issued_parity[s], nullptr, nullptr, 0, 200000000ull);
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        // The issuing thread is the critical path, so every descriptor is a
        // base plus integer offsets: the start-address field is (addr >> 4) in
        // the low 14 bits, and no offset here carries out of it (smem < 256 KB).
        if (lane == 0) {
            uint32_t stage = 0, phase = 0, acc = 0, aphase = 0;
            bool ok = true;
            const uint64_t a_lo0 = tc::smem_u32(sA) >> 4, b_lo0 = tc::smem_u32(sB) >> 4;
            for (int k = 0, tile; ok && (tile = sched_tile(k)) < p.total_tiles; ++k) {
                int mt, nt;
                const Problem &P = p.prob[locate(p, tile, mt, nt)];
                if (!tc::mbar_wait(&tempty[acc], aphase ^ 1, p.ctrl, abort_flag, 0x102)) break;
                tc::tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                const uint32_t idesc =
                    tc::idesc_f16kind_f32(p.fmt, BM, BN, P.a_mn_major, P.b_mn_major);
                const uint64_t a_hi = operand_desc(0, P.a_mn_major, 0);  // address field 0
                const uint64_t b_hi = operand_desc(0, P.b_mn_major, 0);
                const uint32_t a_k = P.a_mn_major ? 2048 >> 4 : 32 >> 4;  // per K=16 step
                const uint32_t b_k = P.b_mn_major ? 2048 >> 4 : 32 >> 4;
                uint32_t accumulate = 0;
                for (int sg = 0; ok && sg < P.nseg; ++sg) {
                    const int nkb = P.seg[sg].nkb;
                    for (int kb = 0; kb < nkb; ++kb) {
                        if (!tc::mbar_wait(&full[stage], phase, p.ctrl, abort_flag, 0x103)) {
                            ok = false;
                            break;
                        }
                        tc::tc_fence_after();
                        const uint64_t ad = a_hi | (a_lo0 + stage * (A_BYTES >> 4));
                        const uint64_t bd = b_hi | (b_lo0 + stage * (B_BYTES >> 4));
                        tc::mma_bf16(d, ad, bd, idesc, accumulate);
                        tc::mma_bf16(d, ad + a_k, bd + b_k, idesc, 1);
                        tc::mma_bf16(d, ad + 2 * a_k, bd + 2 * b_k, idesc, 1);
                        tc::mma_bf16(d, ad + 3 * a_k, bd + 3 * b_k, idesc, 1);
                        accumulate = 1;
                        tc::mma_commit(&empty[stage]);
                        if (++stage == STAGES) stage = 0, phase ^= 1;
                    }
                }
                if (!ok) break;
                if (accumulate) tc::mma_commit(&tfull[acc]);
                else tc::mbar_arrive(&tfull[acc]);  // empty K: nothing to wait for
                acc ^= 1;
                if (acc == 0) aphase ^= 1;
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may read
        uint32_t acc = 0, aphase = 0;
        for (int k = 0, tile; (tile = sched_tile(k)) < p.total_tiles; ++k) {
            int mt, nt;
            const Problem &P = p.prob[locate(p, tile, mt, nt)];
            const bool w = tc::mbar_wait(&tfull[acc], aphase, p.ctrl, abort_flag, 0x104);
            if (!__all_sync(0xffffffffu, w)) break;  // the whole warp leaves together
            tc::tc_fence_after();
            int nk = 0;
            for (int sg = 0; sg < P.nseg; ++sg) nk += P.seg[sg].nkb;
            const int m = mt * BM + q * 32 + lane;
            const int nbase = nt * BN;
            const bool vec = ((P.ldo & 3) == 0) && ((P.out_col0 & 3) == 0) &&
                             ((((uintptr_t)P.out) & 15) == 0);
            // 32-byte stores when rows and the base are 32-byte aligned: each
            // store fills a whole sector instead of half of one
            const bool vec8 = ((P.ldo & 7) == 0) && ((P.out_col0 & 7) == 0) &&
                              ((((uintptr_t)P.out) & 31) == 0);
            for (int c0 = 0; c0 < BN; c0 += 32) {
                if (nbase + c0 >= P.N) break;  // warp-uniform
                uint32_t r[32];
                tc::tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN + c0, r);
                tc::tmem_ld_wait();
                if (m < P.M) {
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int n = nbase + c0 + j;
                        float x = nk ? __uint_as_float(r[j]) : 0.f;
                        if (P.bias && n < P.N) {
                            const unsigned short bb = static_cast<const unsigned short *>(P.bias)[n];
                            x += p.fmt ? __bfloat162float(__ushort_as_bfloat16(bb))
                                       : __half2float(__ushort_as_half(bb));
                        }
                        v[j] = x;
                    }
                    float *orow = P.out + (long long)m * P.ldo + P.out_col0 + nbase + c0;
                    const bool full = nbase + c0 + 32 <= P.N;
                    if (P.accumulate) {
                        if (vec && full) {
#pragma unroll
                            for (int j = 0; j < 32; j += 4) {
                                const float4 o = *reinterpret_cast<const float4 *>(orow + j);
                                v[j] += o.x; v[j + 1] += o.y; v[j + 2] += o.z; v[j + 3] += o.w;
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (nbase + c0 + j < P.N) v[j] += orow[j];
                        }
                    }
                    if (vec8 && full) {
#pragma unroll
                        for (int j = 0; j < 32; j += 8) tc::st_global_v8(orow + j, v + j);
                    } else if (vec && full) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4 *>(orow + j) =
                                make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (nbase + c0 + j < P.N) orow[j] = v[j];
                    }
                }
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
            acc ^= 1;
            if (acc == 0) aphase ^= 1;
        }
    }

    tc::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc::tc_fence_after();
        tc::tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace tcg
}  // namespace lstm
