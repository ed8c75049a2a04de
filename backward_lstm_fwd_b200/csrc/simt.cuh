// simt.cuh -- CUDA-core (FFMA) kernels of the LSTM forward pass and BPTT.
//
// These kernels compute in exact fp32 (fp32 accumulate of products of the
// stored operands).  They are the path for the fp32 compute type, whose 1e-4
// tolerance rules out TF32 tensor-core products, and for shapes off the
// tensor-core tile grid.  One generic tiled GEMM (64x64 tile, 16-deep K slab,
// 256 threads, 4x4 outputs per thread) is specialised by operand accessors and
// fused epilogues:
//   input projection   Gx = X W_x^T + b                (forward-formula table)
//   recurrent step     pre = Gx_t + h_{t-1} W_h^T, gate nonlinearities and the
//                      c/h update fused in the epilogue
//   backward step      delta h_t = dy_t + W_h^T dG_{t+1} fused with backward
//                      steps 1-3 and 5 (delta c, dG_t, delta c_prev)
//   dW                 dG^T [h_prev | x]               (backward step 4)
//   dx                 dG W_x                          (x-part of step 5)
#pragma once

#include "common.cuh"

namespace lstm {
namespace simt {

constexpr int TM = 64, TN = 64, TK = 16, NTHR = 256;

// C[m, n] = sum_k A(m, k) B(k, n) for a 64x64 tile, handed to ep(m, n0, acc[4])
// for the four consecutive columns n0..n0+3 a thread owns.  A_KC / B_KC say
// whether the operand is contiguous along k (picks the coalesced load order).
// Split K (gridDim.z > 1): block z sums k in [z * Kc, min(K, (z + 1) * Kc)).
template <bool A_KC, bool B_KC, class AL, class BL, class EP>
__global__ void __launch_bounds__(NTHR)
gemm_kernel(int M, int N, int K, int Kc, AL A, BL Bm, EP ep) {
    __shared__ __align__(16) float As[TK][TM + 4];
    __shared__ __align__(16) float Bs[TK][TN + 4];
    const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
    const int m0 = blockIdx.x * TM, n0 = blockIdx.y * TN;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // Software pipeline: the next K slab's operands are loaded from global
    // memory into registers while the current slab is multiplied out of
    // shared memory, so each slab's load latency overlaps the previous
    // slab's FMAs instead of following them.
    constexpr int EA = (TM * TK) / NTHR, EB = (TN * TK) / NTHR;
    const int kbeg = (int)blockIdx.z * Kc, kend = min(K, kbeg + Kc);
    float ra[EA], rb[EB];
    auto load = [&](int k0) {
#pragma unroll
        for (int e = 0; e < EA; ++e) {
            const int idx = tid + e * NTHR;
            int mm, kk;
            if (A_KC) { kk = idx % TK; mm = idx / TK; }
            else      { mm = idx % TM; kk = idx / TM; }
            const int m = m0 + mm, k = k0 + kk;
            ra[e] = (m < M && k < kend) ? A(m, k) : 0.f;
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            const int idx = tid + e * NTHR;
            int nn, kk;
            if (B_KC) { kk = idx % TK; nn = idx / TK; }
            else      { nn = idx % TN; kk = idx / TN; }
            const int n = n0 + nn, k = k0 + kk;
            rb[e] = (n < N && k < kend) ? Bm(k, n) : 0.f;
        }
    };
    auto store = [&]() {
#pragma unroll
        for (int e = 0; e < EA; ++e) {
            const int idx = tid + e * NTHR;
            if (A_KC) As[idx % TK][idx / TK] = ra[e];
            else      As[idx / TM][idx % TM] = ra[e];
        }
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            const int idx = tid + e * NTHR;
            if (B_KC) Bs[idx % TK][idx / TK] = rb[e];
            else      Bs[idx / TN][idx % TN] = rb[e];
        }
    };
    if (kbeg < kend) load(kbeg);
    for (int k0 = kbeg; k0 < kend; k0 += TK) {
        store();
        __syncthreads();
        if (k0 + TK < kend) load(k0 + TK);
#pragma unroll
        for (int kk = 0; kk < TK; ++kk) {
            // this thread's rows 4 ty .. 4 ty + 3 and columns 4 tx .. 4 tx + 3:
            // one 16-byte shared load for each operand per k
            const float4 av = *reinterpret_cast<const float4 *>(&As[kk][4 * ty]);
            const float a[4] = {av.x, av.y, av.z, av.w};
            const float4 bv = *reinterpret_cast<const float4 *>(&Bs[kk][4 * tx]);
            const float b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + 4 * ty + i;
        if (m < M) ep(m, n0 + 4 * tx, acc[i]);
    }
}

// splits > 1: K split into that many slabs of whole TK blocks, one grid layer
// each (the epilogue sees blockIdx.z; see EpPart).
template <bool A_KC, bool B_KC, class AL, class BL, class EP>
inline cudaError_t gemm(int M, int N, int K, AL A, BL Bm, EP ep, cudaStream_t s,
                        int splits = 1) {
    if (M <= 0 || N <= 0) return cudaSuccess;
    const int Kc = splits > 1 ? ((K + splits - 1) / splits + TK - 1) / TK * TK : K;
    dim3 grid((M + TM - 1) / TM, (N + TN - 1) / TN, splits > 1 ? splits : 1);
    if (grid.y > 65535u || grid.z > 64u) return cudaErrorInvalidConfiguration;
    gemm_kernel<A_KC, B_KC><<<grid, NTHR, 0, s>>>(M, N, K, Kc, A, Bm, ep);
    note_launch();
    return cudaGetLastError();
}

// ---------------------------------------------------------------- accessors
// Row-major matrix view p[i * ld + j].
template <class T> struct RowMajor {
    const T *p; long long ld;
    __device__ float operator()(int i, int j) const { return to_f(p[(long long)i * ld + j]); }
};
// Transposed view: element (i, j) is p[j * ld + i].
template <class T> struct ColMajor {
    const T *p; long long ld;
    __device__ float operator()(int i, int j) const { return to_f(p[(long long)j * ld + i]); }
};

// B operand of the input projection: (k, n) -> W[n][H + k]  (W_x^T).
template <class T> struct WxT {
    const T *W; int H, I;
    __device__ float operator()(int k, int n) const {
        return to_f(W[(long long)n * (H + I) + H + k]);
    }
};

// B operand of the recurrent step with gate-interleaved columns: logical column
// q = 4 j + g maps to W row g*H + j, so one thread's four columns are the four
// gates of hidden unit j.  (k, q) -> W_h[g*H + j][k].
template <class T> struct WhT4 {
    const T *W; int H, I;
    __device__ float operator()(int k, int q) const {
        const int j = q >> 2, g = q & 3;
        return to_f(W[((long long)g * H + j) * (H + I) + k]);
    }
};

// h_{t-1} for step t: y[t-1] for t > 0, initH (or zeros) for t = 0.
template <class T> struct Hprev {
    const T *hp; int H;  // hp = y + (t-1)*B*H or h0 (may be NULL)
    __device__ float operator()(int n, int k) const {
        return hp ? to_f(hp[(long long)n * H + k]) : 0.f;
    }
};

// z-rows for dW: row r = t*B + n, column c < H -> h_{t-1}[n][c], else x_t[n][c-H].
template <class T> struct Zrows {
    const T *x, *y, *h0; int B, I, H;
    // reverse direction: h_prev of time t is y[t+1], and h0 at the last time
    // (whose rows start at last0 = (T-1) * B)
    bool reverse = false;
    long long last0 = 0;
    __device__ float operator()(int r, int c) const {
        if (c < H) {
            if (!reverse) {
                if (r < B) return h0 ? to_f(h0[(long long)r * H + c]) : 0.f;
                return to_f(y[(long long)(r - B) * H + c]);
            }
            if (r >= last0) return h0 ? to_f(h0[(long long)(r - last0) * H + c]) : 0.f;
            return to_f(y[(long long)(r + B) * H + c]);
        }
        return to_f(x[(long long)r * I + (c - H)]);
    }
};

// ---------------------------------------------------------------- epilogues
// Gx[r][n] = acc + b[n]  (input projection with the bias fused).
template <class T> struct EpGx {
    float *Gx; const T *b; int N;
    __device__ void operator()(int m, int n0, const float *acc) const {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int n = n0 + c;
            if (n < N) Gx[(long long)m * N + n] = acc[c] + (b ? to_f(b[n]) : 0.f);
        }
    }
};

// Recurrent forward step t (forward-formula table): acc holds W_h h_{t-1} for
// gates i, f, g, o of hidden unit j = n0 / 4 of sequence m.
template <class T> struct EpFwdStep {
    const float *Gx;            // [T*B][4H], row t*B + m
    const float *cprev;         // cells[t-1] or c0 (may be NULL), [B][H]
    T *y; T *gates; float *cells;  // step-t slices: [B][H], [B][4H], [B][H]
    int H;
    // variable length: mask[t] [B][H] (1 = real step, 0 = padding, which keeps
    // h_{t-1} = y[t-1] or h0, and c_{t-1}); NULL = every step real
    const T *mask = nullptr;
    const T *hprev = nullptr;
    // row block of the forget gate: 1 for gate_order "ifjo", 2 for "ijfo"
    // (the candidate j = g takes the other of blocks 1 and 2)
    int fb = 1;
    __device__ void operator()(int m, int q0, const float *acc) const {
        const int j = q0 >> 2;
        if (j >= H) return;
        const int gb = 3 - fb;
        const float *gx = Gx + (long long)m * 4 * H;
        const float ig = sigmoidf_(acc[0] + gx[j]);
        const float fg = sigmoidf_(acc[fb] + gx[fb * H + j]);
        const float gg = tanhf_(acc[gb] + gx[gb * H + j]);
        const float og = sigmoidf_(acc[3] + gx[3 * H + j]);
        const float cp = cprev ? cprev[(long long)m * H + j] : 0.f;
        float c = fg * cp + ig * gg;
        float h = og * tanhf_(c);
        if (mask) {
            const float mk = to_f(mask[(long long)m * H + j]);
            const float hp = hprev ? to_f(hprev[(long long)m * H + j]) : 0.f;
            c = mk * c + (1.f - mk) * cp;
            h = mk * h + (1.f - mk) * hp;
        }
        T *gt = gates + (long long)m * 4 * H;
        gt[j] = from_f<T>(ig);
        gt[fb * H + j] = from_f<T>(fg);
        gt[gb * H + j] = from_f<T>(gg);
        gt[3 * H + j] = from_f<T>(og);
        cells[(long long)m * H + j] = c;
        y[(long long)m * H + j] = from_f<T>(h);
    }
};

// Backward step t ("backward algorithm", steps 1, 2, 3 and 5): acc holds
// W_h^T dG_{t+1} for hidden units n0..n0+3 of sequence m (zero at t = T-1).
template <class T> struct EpBwdStep {
    const T *dy;        // dy[t] slice [B][H] or NULL
    const T *dh_in;     // dhT [B][H] at t = T-1 (else NULL: use acc)
    const float *dc_in; // dcT at t = T-1, else delta c_next buffer; may be NULL
    const T *gates;     // gates[t] [B][4H]
    const float *cells; // cells[t] [B][H]
    const float *cprev; // cells[t-1] or c0 or NULL
    T *dG;              // dG[t] [B][4H]
    float *dc_out;      // delta c_prev [B][H]
    int H; bool use_acc;
    // variable length: mask[t] [B][H] (NULL = every step real); padding passes
    // the share (1 - m) of delta h to h_{t-1} through dhp_out (read back as
    // dhp_in one step earlier) and of delta c_next to c_{t-1}
    const T *mask = nullptr;
    const float *dhp_in = nullptr;
    float *dhp_out = nullptr;
    int fb = 1;  // row block of the forget gate (2 for gate_order "ijfo")
    __device__ void operator()(int m, int n0, const float *acc) const {
        const int gb = 3 - fb;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const int j = n0 + c;
            if (j >= H) continue;
            const long long o = (long long)m * H + j;
            float dh = dy ? to_f(dy[o]) : 0.f;                       // step 1
            dh += use_acc ? acc[c] : (dh_in ? to_f(dh_in[o]) : 0.f);
            if (dhp_in) dh += dhp_in[o];
            float dcn = dc_in ? dc_in[o] : 0.f;
            float mk = 1.f;
            // (__fmul_rn: no contraction into the sums below, so that m = 1
            // rounds exactly as an unmasked call does)
            if (mask) {
                mk = to_f(mask[o]);
                dhp_out[o] = __fmul_rn(1.f - mk, dh);
                dh = __fmul_rn(dh, mk);
            }
            const float dc_pass = __fmul_rn(1.f - mk, dcn);
            dcn = __fmul_rn(dcn, mk);
            const T *g4 = gates + (long long)m * 4 * H;
            const float ig = to_f(g4[j]), fg = to_f(g4[fb * H + j]);
            const float gg = to_f(g4[gb * H + j]), og = to_f(g4[3 * H + j]);
            const float ct = cells[o];
            const float cp = cprev ? cprev[o] : 0.f;
            const float tc = tanhf_(ct);
            const float dc = dh * og * (1.f - tc * tc) + dcn;          // step 2
            const float d_o = dh * tc * og * (1.f - og);               // step 3
            const float d_g = dc * ig * (1.f - gg * gg);
            const float d_i = dc * gg * ig * (1.f - ig);
            const float d_f = dc * cp * fg * (1.f - fg);
            T *d4 = dG + (long long)m * 4 * H;
            d4[j] = from_f<T>(d_i);
            d4[fb * H + j] = from_f<T>(d_f);
            d4[gb * H + j] = from_f<T>(d_g);
            d4[3 * H + j] = from_f<T>(d_o);
            dc_out[o] = dc * fg + dc_pass;                             // step 5
        }
    }
};

// Plain float store of the GEMM result: out[m][n], row stride N (plus
// add[m][n] when add is not NULL).
struct EpStore {
    float *out; int N;
    const float *add = nullptr;
    __device__ void operator()(int m, int n0, const float *acc) const {
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (n0 + c < N)
                out[(long long)m * N + n0 + c] =
                    acc[c] + (add ? add[(long long)m * N + n0 + c] : 0.f);
    }
};

// Partial product of K split z (blockIdx.z) of a split-K GEMM:
// part[z][m][n], row stride N, MN floats per split.
struct EpPart {
    float *part; int N; long long MN;
    __device__ void operator()(int m, int n0, const float *acc) const {
        float *o = part + (long long)blockIdx.z * MN + (long long)m * N;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (n0 + c < N) o[n0 + c] = acc[c];
    }
};

// out[i] = sum over the S splits of part[z][i], in split order.
__global__ void sum_splits(const float *part, int S, long long MN, float *out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= MN) return;
    float v = 0.f;
    for (int z = 0; z < S; ++z) v += part[(long long)z * MN + i];
    out[i] = v;
}

// ----------------------------------------------------------- db (step 4)
// Column sums of dG [R][N] in two deterministic passes: per-chunk partials,
// then a sum over chunks.
template <class T>
__global__ void colsum_partial(const T *dG, int R, int N, int rows_per_chunk, float *part) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    const int chunk = blockIdx.y;
    if (n >= N) return;
    const int r0 = chunk * rows_per_chunk;
    const int r1 = min(R, r0 + rows_per_chunk);
    float s = 0.f;
    for (int r = r0; r < r1; ++r) s += to_f(dG[(long long)r * N + n]);
    part[(long long)chunk * N + n] = s;
}

__global__ void colsum_final(const float *part, int chunks, int N, float *out) {
    const int n = blockIdx.x * blockDim.x + threadIdx.x;
    if (n >= N) return;
    float s = 0.f;
    for (int c = 0; c < chunks; ++c) s += part[(long long)c * N + n];
    out[n] = s;
}

// out[i] = float(in[i]) (or 0 when in is NULL).
template <class T>
__global__ void to_float_copy(const T *in, float *out, long long n) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = in ? to_f(in[i]) : 0.f;
}

// float -> compute type (the gradient at a layer's outputs, handed to the
// layer below it as its dy)
template <class T>
__global__ void from_float_copy(const float *in, T *out, long long n) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = from_f<T>(in[i]);
}

template <class T>
__global__ void copy_or_zero(const T *in, T *out, long long n) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i < n) out[i] = in ? in[i] : from_f<T>(0.f);
}

}  // namespace simt
}  // namespace lstm
