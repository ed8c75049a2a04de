// common.cuh -- element conversions, activations and the workspace control
// block shared by every liblstm kernel.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace lstm {

// Host-side count of kernel launches issued by the library (diagnostics).
inline std::atomic<long long> &launch_counter() {
    static std::atomic<long long> n{0};
    return n;
}
inline void note_launch(long long k = 1) { launch_counter().fetch_add(k); }

// ---------------------------------------------------------------- elements
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f(__half v) { return __half2float(v); }

template <class T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
    return __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }

// 16-bit compute types of the tensor-core kernels: bf16 and fp16 (IEEE
// binary16).  kFmt is the operand format of tcgen05.mma kind::f16 (0 = f16,
// 1 = bf16); x8 / f32x8 convert 8 packed elements (one 16-byte vector).
template <class E> struct Elem;
template <> struct Elem<__nv_bfloat16> {
    static constexpr uint32_t kFmt = 1;
    typedef __nv_bfloat162 E2;
    __device__ static __forceinline__ float2 to_f2(E2 v) { return __bfloat1622float2(v); }
    __device__ static __forceinline__ E2 from_f2(float a, float b) { return __floats2bfloat162_rn(a, b); }
};
template <> struct Elem<__half> {
    static constexpr uint32_t kFmt = 0;
    typedef __half2 E2;
    __device__ static __forceinline__ float2 to_f2(E2 v) { return __half22float2(v); }
    __device__ static __forceinline__ E2 from_f2(float a, float b) { return __floats2half2_rn(a, b); }
};

template <class E> __device__ __forceinline__ void x8_to_f32(const uint4 &v, float (&f)[8]) {
    const typename Elem<E>::E2 *h = reinterpret_cast<const typename Elem<E>::E2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 x = Elem<E>::to_f2(h[i]);
        f[2 * i] = x.x;
        f[2 * i + 1] = x.y;
    }
}
template <class E> __device__ __forceinline__ uint4 f32x8_to(const float (&f)[8]) {
    uint4 v;
    typename Elem<E>::E2 *h = reinterpret_cast<typename Elem<E>::E2 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = Elem<E>::from_f2(f[2 * i], f[2 * i + 1]);
    return v;
}

// ------------------------------------------------------------- activations
// Gate nonlinearities of the forward-formula table ("SingleLayerLstmGrad"):
// sigma for the input, forget and output gates, tanh for the candidate state
// and for the cell state feeding h_t.  expf / tanhf are CUDA's own functions.
__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }
__device__ __forceinline__ float tanhf_(float a) { return tanhf(a); }

// ------------------------------------------------------- workspace control
// The first 256 bytes of every workspace.  `status` is sticky: kernels only
// ever set it, and lstm_status() reads and clears it.  Barrier counters are
// zeroed at the start of every call.
struct Ctrl {
    unsigned int status;     // 0 or an LSTM_ERR_* code
    unsigned int fail_site;  // which wait gave up (for diagnostics)
    unsigned int pad[14];
    unsigned int bar[48];    // grid-barrier counters
};
static_assert(sizeof(Ctrl) == 256, "control block is 256 bytes");

constexpr size_t kCtrlBytes = 256;

__host__ __device__ __forceinline__ size_t align_up(size_t v, size_t a) {
    return (v + a - 1) / a * a;
}

}  // namespace lstm
