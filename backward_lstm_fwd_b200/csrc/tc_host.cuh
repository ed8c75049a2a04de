// tc_host.cuh -- host side of the tcgen05 GEMM core: TMA tensor-map encoding
// (reached through cudaGetDriverEntryPoint, so the library needs no libcuda
// link), problem-table construction and the persistent launch.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstring>

#include "tc_gemm.cuh"

namespace lstm {
namespace tcg {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// 2-D tensor map of 16-bit elements (bf16 by default, or fp16) with 128-byte
// swizzle: `inner` contiguous elements per row, `outer` rows `row_bytes`
// apart, boxes of box_inner x box_outer.  Reads outside the extents return
// zeros.
inline bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || inner == 0 || outer == 0) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Operand view for a problem: a row-major matrix of 16-bit elements, `rows` x
// `cols` (row stride ld elements).  As a K-major operand the rows are M (or N)
// and the columns K; as an MN-major operand the rows are K and the columns M / N.
struct View {
    const void *p;
    long long rows, cols, ld;
};

// the tensor-map element type of operand format fmt (0 = fp16, 1 = bf16)
inline CUtensorMapDataType map_type(uint32_t fmt) {
    return fmt ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
}

inline bool map_for(CUtensorMap *m, const View &v, int mn_major, int mn_tile, uint32_t fmt) {
    return mn_major ? make_map(m, v.p, v.cols, v.rows, v.ld * 2, 64, BK, map_type(fmt))
                    : make_map(m, v.p, v.cols, v.rows, v.ld * 2, BK, mn_tile, map_type(fmt));
}

struct Builder {
    Params P;
    int nmaps = 0;
    bool ok = true;
    // fmt: operand format of the launch, 0 = fp16, 1 = bf16
    Builder(Ctrl *ctrl, uint32_t fmt = 1) {
        memset(&P, 0, sizeof(P));
        P.ctrl = ctrl;
        P.fmt = fmt;
    }
    int add_map(const View &v, int mn_major, int mn_tile) {
        if (nmaps >= MAX_MAPS) { ok = false; return 0; }
        if (!map_for(&P.maps[nmaps], v, mn_major, mn_tile, P.fmt)) ok = false;
        return nmaps++;
    }
    Problem &add_problem(int M, int N, int a_mn, int b_mn, float *out, long long ldo,
                         int out_col0, const void *bias) {
        if (P.nprob >= MAX_PROB) { ok = false; return P.prob[0]; }
        Problem &q = P.prob[P.nprob++];
        memset(&q, 0, sizeof(q));
        q.M = M; q.N = N; q.a_mn_major = a_mn; q.b_mn_major = b_mn;
        q.out = out; q.ldo = ldo; q.out_col0 = out_col0; q.bias = bias; q.accumulate = 0;
        return q;
    }
    static void add_seg(Problem &q, int a_map, int a_k0, int b_map, int b_k0, long long K) {
        Seg &s = q.seg[q.nseg++];
        s.a_map = a_map; s.b_map = b_map; s.a_k0 = a_k0; s.b_k0 = b_k0;
        s.nkb = (int)((K + BK - 1) / BK);
    }
    void finalize() {
        int t = 0;
        for (int i = 0; i < P.nprob; ++i) {
            Problem &q = P.prob[i];
            const int tm = (q.M + BM - 1) / BM;
            q.tiles_n = (q.N + BN - 1) / BN;
            q.tile_begin = t;
            t += tm * q.tiles_n;
            q.tile_end = t;
        }
        P.total_tiles = t;
        // unused map slots: copy map 0 so that every prefetched descriptor is valid
        for (int i = nmaps; i < MAX_MAPS && nmaps > 0; ++i) P.maps[i] = P.maps[0];
    }
};

inline int sm_count() {
    static int n = 0;
    if (!n) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 1;
    }
    return n;
}

inline cudaError_t launch(Builder &b, cudaStream_t s, int max_ctas = 0) {
    b.finalize();
    if (b.P.total_tiles == 0) return cudaSuccess;
    static bool attr = false;
    if (!attr) {
        cudaError_t e = cudaFuncSetAttribute(gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr = true;
    }
    int grid = std::min(b.P.total_tiles, max_ctas > 0 ? max_ctas : sm_count());
    gemm_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(b.P);
    note_launch();
    return cudaGetLastError();
}

}  // namespace tcg
}  // namespace lstm
