// eqlin_prep.cuh -- weight pre-transform (run once per weight update) and the fp32
// fused forward.
//
// Page "Flash EQ-Linear: Accelerating Equivariant Linear Layers via Group-wise
// Discrete Fourier Transform", section "Enfoque Algoritmico": in the frequency
// domain the group convolution is a pointwise product, so the weights are moved to
// the frequency domain once (W^_k = sum_m w_m exp(-2 pi i m k / G), k = 0..G/2) and
// reused by every forward.  Layouts: eqlin_layout.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

#include "eqlin_layout.h"
#include "group_dft.cuh"
#include "io16.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

template <typename T>
__device__ __forceinline__ double load_as_double(const T* p, size_t i);
template <>
__device__ __forceinline__ double load_as_double<float>(const float* p, size_t i) {
    return static_cast<double>(p[i]);
}
template <>
__device__ __forceinline__ double load_as_double<__nv_bfloat16>(const __nv_bfloat16* p, size_t i) {
    return static_cast<double>(__bfloat162float(p[i]));
}
template <>
__device__ __forceinline__ double load_as_double<__half>(const __half* p, size_t i) {
    return static_cast<double>(__half2float(p[i]));
}

// One thread per (o, i) of the operator: real DFT of its filter f[o, i, :] in
// float64, scaled for the folded inverse (1/G real planes, 2/G complex planes),
// stored to w_f32[p][i][o] and, when w_f64 is not null, to w_f64[p][i][o].  Thread
// (o, i = 0) also converts bias[o] (0 when bias is null) to bias_f32[o] and, when
// requested, bias_f64[o].
//
// The operator is [Cout, Cin] with filter f = w (w is [Cout, Cin, G]) when
// `adjoint` is false.  With `adjoint` true it is the input gradient of the layer:
// dx[n,i,h] = sum_{o,g} w[o,i,(g-h) mod G] dy[n,o,g] is the same block-circulant
// product with the channel axes swapped and the filter reflected,
// f[i, o, m] = w[o, i, (-m) mod G]; then Cout and Cin here are the layer's Cin and
// Cout and w is still the layer's [Cin_here, Cout_here, G] weight.
template <typename T>
__global__ void eqlin_prep_freq_kernel(const T* __restrict__ w, const T* __restrict__ bias, int Cout,
                                       int Cin, int G, float* __restrict__ w_f32,
                                       float* __restrict__ bias_f32, double* __restrict__ w_f64,
                                       double* __restrict__ bias_f64, bool adjoint = false) {
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(Cout) * Cin) return;
    const int o = static_cast<int>(idx / Cin), i = static_cast<int>(idx % Cin);
    const size_t base = adjoint ? (static_cast<size_t>(i) * Cout + o) * G : static_cast<size_t>(idx) * G;
    for (int p = 0; p < G; ++p) {
        const int k = p == 0 ? 0 : (p == 1 ? G / 2 : p / 2);
        const bool imag = p >= 2 && (p & 1);
        const double scale = (p < 2 ? 1.0 : 2.0) / G;
        double acc = 0.0;
        for (int m = 0; m < G; ++m) {
            double s, c;
            sincospi(2.0 * static_cast<double>((m * k) % G) / G, &s, &c);
            const int src = adjoint ? (G - m) % G : m;
            acc += load_as_double(w, base + src) * (imag ? -s : c);
        }
        const size_t dst = (static_cast<size_t>(p) * Cin + i) * Cout + o;
        w_f32[dst] = static_cast<float>(scale * acc);
        if (w_f64 != nullptr) w_f64[dst] = scale * acc;
    }
    if (i == 0) {
        const double b = bias != nullptr ? load_as_double(bias, o) : 0.0;
        bias_f32[o] = static_cast<float>(b);
        if (bias_f64 != nullptr) bias_f64[o] = b;
    }
}

// One thread per element of the 16-bit (T16: bf16 or fp16) tensor-core image (see
// eqlin_layout.h).  `rows` rows per sub-block; output chunk oc covers o = oc*128 + r.
template <class T16>
__global__ void eqlin_prep_image_kernel(const float* __restrict__ w_f32, int Cout, int Cin, int G,
                                        int nK, int rows, size_t n_elems, uint8_t* __restrict__ img) {
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n_elems) return;
    const int col = static_cast<int>(idx % kChunkK);
    const int r = static_cast<int>((idx / kChunkK) % rows);
    const size_t sub = idx / (static_cast<size_t>(kChunkK) * rows);
    const int p = static_cast<int>(sub % G);
    const int c = static_cast<int>((sub / G) % nK);
    const int oc = static_cast<int>(sub / (static_cast<size_t>(G) * nK));
    const int o = oc * kMmaM + r;
    const int i = c * kChunkK + col;
    float v = 0.0f;
    if (o < Cout && i < Cin) v = w_f32[(static_cast<size_t>(p) * Cin + i) * Cout + o];
    *reinterpret_cast<T16*>(img + image_offset(sub, rows, r, col)) = Io16<T16>::from_float(v);
}

// Image for the tokens-on-M kernel (layout: image_offset_k16 over the weight slots,
// tm_weight_slots).  `rows` rows per sub-block; output chunk oc covers o = oc*rows + r.
template <class T16>
__global__ void eqlin_prep_image_k16_kernel(const float* __restrict__ w_f32, int Cout, int Cin, int G,
                                            int nK, int rows, size_t n_elems, uint8_t* __restrict__ img) {
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= n_elems) return;
    const int SL = tm_weight_slots(G);
    const int col = static_cast<int>(idx % kChunkK16);
    const int r = static_cast<int>((idx / kChunkK16) % rows);
    const size_t sub = idx / (static_cast<size_t>(kChunkK16) * rows);
    const int slot = static_cast<int>(sub % SL);
    const int c = static_cast<int>((sub / SL) % nK);
    const int oc = static_cast<int>(sub / (static_cast<size_t>(SL) * nK));
    const int o = oc * rows + r;
    const int i = c * kChunkK16 + col;
    float sign = 1.0f;
    const int p = tm_pair_slots(G) ? pair_slot_plane(slot, &sign) : slot;
    float v = 0.0f;
    if (o < Cout && i < Cin) v = sign * w_f32[(static_cast<size_t>(p) * Cin + i) * Cout + o];
    *reinterpret_cast<T16*>(img + image_offset_k16(sub, rows, r, col)) = Io16<T16>::from_float(v);
}

// ------------------------------------------------------------------ fp32 path
// Fused forward for fp32 I/O on CUDA cores.  The tensor-core kinds that take fp32
// operands round them to tf32 (10-bit mantissa), far from a 1e-5 bound, so this
// path keeps x, the spectra, the weights and the accumulation in float64 and
// rounds once, when y is stored (elementwise relative error ~2^-24).
// Block = 8 warps; block (bx, by) handles tokens [8 bx, 8 bx + 8) and outputs
// [32 by, 32 by + 32); warp = token, lane = output channel.
constexpr int kF32Tokens = 8;
constexpr int kF32Threads = 256;

template <int G>
__global__ void __launch_bounds__(kF32Threads)
    eqlin_fwd_f32_kernel(const float* __restrict__ x, const double* __restrict__ w_f64,
                         const double* __restrict__ bias_f64, float* __restrict__ y, long long N,
                         int Cin, int Cout, int act) {
    extern __shared__ double xs[];  // [kF32Tokens][G][Cin] spectrum of the block's tokens
    // launched as a programmatic dependent: the next kernel of the stream may start its
    // blocks as these exit, and x and y are touched only once the previous one has completed
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();
    const long long n0 = static_cast<long long>(blockIdx.x) * kF32Tokens;
    for (int idx = threadIdx.x; idx < kF32Tokens * Cin; idx += kF32Threads) {
        const int t = idx / Cin, i = idx % Cin;
        const long long n = n0 + t;
        double v[G], pl[G];
#pragma unroll
        for (int h = 0; h < G; ++h) v[h] = n < N ? static_cast<double>(x[(n * Cin + i) * G + h]) : 0.0;
        rdft_planes<G, double>(v, pl);
#pragma unroll
        for (int p = 0; p < G; ++p) xs[(t * G + p) * Cin + i] = pl[p];
    }
    __syncthreads();
    const int t = threadIdx.x >> 5;
    const long long n = n0 + t;
    const int o = blockIdx.y * 32 + (threadIdx.x & 31);
    if (n >= N || o >= Cout) return;
    double z[G];
#pragma unroll
    for (int p = 0; p < G; ++p) z[p] = 0.0;
    const double* xt = xs + t * G * Cin;
    for (int i = 0; i < Cin; ++i) {
        double xv[G], wv[G];
#pragma unroll
        for (int p = 0; p < G; ++p) {
            xv[p] = xt[p * Cin + i];
            wv[p] = w_f64[(static_cast<size_t>(p) * Cin + i) * Cout + o];
        }
        z[0] = fma(wv[0], xv[0], z[0]);
        z[1] = fma(wv[1], xv[1], z[1]);
#pragma unroll
        for (int k = 1; k < G / 2; ++k) {
            const int pr = 2 * k, pi = 2 * k + 1;
            z[pr] = fma(wv[pr], xv[pr], fma(-wv[pi], xv[pi], z[pr]));
            z[pi] = fma(wv[pi], xv[pr], fma(wv[pr], xv[pi], z[pi]));
        }
    }
    z[0] += bias_f64[o];
    double yv[G];
    RealIdft<G, double>::run(z, yv);
    if (act == kActGelu) {
#pragma unroll
        for (int g = 0; g < G; ++g) yv[g] = gelu(yv[g]);
    }
    float* dst = y + (n * Cout + o) * G;
    if constexpr (G % 4 == 0) {
#pragma unroll
        for (int g = 0; g < G; g += 4) {
            *reinterpret_cast<float4*>(dst + g) =
                make_float4(static_cast<float>(yv[g]), static_cast<float>(yv[g + 1]),
                            static_cast<float>(yv[g + 2]), static_cast<float>(yv[g + 3]));
        }
    } else {
        *reinterpret_cast<float2*>(dst) = make_float2(static_cast<float>(yv[0]), static_cast<float>(yv[1]));
    }
}

}  // namespace eqlin
