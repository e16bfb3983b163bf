// group_dft.cuh -- register-resident real DFT / inverse real DFT along the group
// axis of C_G, G in {2, 4, 8, 16}, fully unrolled at compile time.
//
// Method: page "Flash EQ-Linear: Accelerating Equivariant Linear Layers via
// Group-wise Discrete Fourier Transform", section "Enfoque Algoritmico": the group
// convolution becomes a pointwise product per frequency after a DFT over G, and
// because inputs and weights are real only the non-redundant half of the spectrum
// (k = 0 .. G/2) is formed.  For p4 the transforms are pure additions and
// subtractions (section "Especializacion para el Grupo de Rotacion p4"); the
// recursion below reproduces that: G = 4 costs 8 add/sub forward, 8 inverse.
//
// T is float or fx2 (bf16 path: one or two transforms at a time) or double (fp32-I/O
// path).
//
// Frequency components are kept in "plane order":
//   plane 0      = Re X_0          (real)
//   plane 1      = Re X_{G/2}      (real, Nyquist)
//   plane 2k     = Re X_k,  plane 2k+1 = Im X_k    for 0 < k < G/2
// Forward sign: X_k = sum_h x_h exp(-2 pi i h k / G), no scaling.
#pragma once

#include <type_traits>
#include <utility>

namespace eqlin {

// cos(2*pi*j/16), exact closed forms: cos(pi/8) = sqrt(2+sqrt(2))/2,
// cos(pi/4) = sqrt(2)/2, cos(3pi/8) = sqrt(2-sqrt(2))/2, rounded to T.
template <typename T = float>
__host__ __device__ constexpr T cos16(int j) {
    constexpr T c1 = static_cast<T>(0.923879532511286756128183189396788933);
    constexpr T c2 = static_cast<T>(0.707106781186547524400844362104849039);
    constexpr T c3 = static_cast<T>(0.382683432365089771728459984030398867);
    j &= 15;
    switch (j) {
        case 0: return T(1);
        case 1: return c1;
        case 2: return c2;
        case 3: return c3;
        case 4: return T(0);
        case 5: return -c3;
        case 6: return -c2;
        case 7: return -c1;
        case 8: return T(-1);
        case 9: return -c1;
        case 10: return -c2;
        case 11: return -c3;
        case 12: return T(0);
        case 13: return c3;
        case 14: return c2;
        default: return c1;
    }
}
// sin(2*pi*j/16) = cos(2*pi*(j-4)/16)
template <typename T = float>
__host__ __device__ constexpr T sin16(int j) { return cos16<T>(j - 4); }

__device__ __forceinline__ float fma_t(float a, float b, float c) { return fmaf(a, b, c); }
__device__ __forceinline__ double fma_t(double a, double b, double c) { return fma(a, b, c); }

// Two fp32 lanes carried together, so that two independent transforms (two tokens or
// two channels) run as one instruction stream on sm_100's packed FP32x2 add, multiply
// and fused multiply-add (__fadd2_rn, __fmul2_rn, __ffma2_rn).  Each lane rounds
// exactly as the scalar float operation would, so results are bit-identical to two
// scalar transforms.
struct fx2 {
    float x, y;
    __host__ __device__ constexpr fx2() : x(0.0f), y(0.0f) {}
    __host__ __device__ constexpr fx2(double v) : x(static_cast<float>(v)), y(static_cast<float>(v)) {}
    __host__ __device__ constexpr fx2(float a, float b) : x(a), y(b) {}
};
__device__ __forceinline__ float2 as_float2(fx2 a) { return make_float2(a.x, a.y); }
__device__ __forceinline__ fx2 as_fx2(float2 a) { return fx2(a.x, a.y); }
__device__ __forceinline__ fx2 operator+(fx2 a, fx2 b) { return as_fx2(__fadd2_rn(as_float2(a), as_float2(b))); }
__device__ __forceinline__ fx2 operator-(fx2 a) { return fx2(-a.x, -a.y); }
// a - b as a + b * (-1): the product is exact, so this rounds like a subtraction
__device__ __forceinline__ fx2 operator-(fx2 a, fx2 b) {
    return as_fx2(__ffma2_rn(as_float2(b), make_float2(-1.0f, -1.0f), as_float2(a)));
}
__device__ __forceinline__ fx2 operator*(fx2 a, fx2 b) { return as_fx2(__fmul2_rn(as_float2(a), as_float2(b))); }
__device__ __forceinline__ fx2& operator+=(fx2& a, fx2 b) { return a = a + b; }
__device__ __forceinline__ fx2& operator-=(fx2& a, fx2 b) { return a = a - b; }
__device__ __forceinline__ fx2 fma_t(fx2 a, fx2 b, fx2 c) {
    return as_fx2(__ffma2_rn(as_float2(a), as_float2(b), as_float2(c)));
}

template <int N, class F, int... Is>
__device__ __forceinline__ void static_for_impl(F&& f, std::integer_sequence<int, Is...>) {
    (f(std::integral_constant<int, Is>{}), ...);
}
// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1 (compile-time indices).
template <int N, class F>
__device__ __forceinline__ void static_for(F&& f) {
    static_for_impl<N>(static_cast<F&&>(f), std::make_integer_sequence<int, N>{});
}

// acc += v * cos(2 pi J / 16) and accI -= v * sin(2 pi J / 16), with the trivial
// angles (multiples of pi/2) done as plain adds.
template <int J, typename T>
__device__ __forceinline__ void twiddle_acc(T v, T& re, T& im) {
    constexpr int j = J & 15;
    if constexpr (j == 0) {
        re += v;
    } else if constexpr (j == 4) {
        im -= v;
    } else if constexpr (j == 8) {
        re -= v;
    } else if constexpr (j == 12) {
        im += v;
    } else {
        re = fma_t(v, cos16<T>(j), re);
        im = fma_t(-v, sin16<T>(j), im);
    }
}

// re*cos(2 pi J/16) - im*sin(2 pi J/16), trivial angles without multiplies.
template <int J, typename T>
__device__ __forceinline__ T rotate_real(T re, T im) {
    constexpr int j = J & 15;
    if constexpr (j == 0) {
        return re;
    } else if constexpr (j == 4) {
        return -im;
    } else if constexpr (j == 8) {
        return -re;
    } else if constexpr (j == 12) {
        return im;
    } else {
        return fma_t(re, cos16<T>(j), -im * sin16<T>(j));
    }
}

// Half-spectrum real DFT of length G: x[G] -> re[G/2+1], im[G/2+1]
// (im[0] and im[G/2] are zero and not written).  Decimation in frequency:
// u_h = x_h + x_{h+G/2} carries the even frequencies (a length-G/2 real DFT),
// v_h = x_h - x_{h+G/2} the odd ones.
template <int G, typename T = float>
struct RealDft {
    static_assert(G >= 4 && (G & (G - 1)) == 0, "G must be a power of two >= 4");
    __device__ __forceinline__ static void run(const T (&x)[G], T (&re)[G / 2 + 1], T (&im)[G / 2 + 1]) {
        constexpr int H = G / 2;
        T u[H], v[H];
#pragma unroll
        for (int h = 0; h < H; ++h) {
            u[h] = x[h] + x[h + H];
            v[h] = x[h] - x[h + H];
        }
        T ure[H / 2 + 1], uim[H / 2 + 1];
        RealDft<H, T>::run(u, ure, uim);
        static_for<H / 2 + 1>([&](auto kk) {
            constexpr int k = decltype(kk)::value;
            re[2 * k] = ure[k];
            if constexpr (k != 0 && 2 * k != H) im[2 * k] = uim[k];
        });
        // odd frequencies k = 1, 3, ..., H-1
        static_for<H / 2>([&](auto jj) {
            constexpr int k = 2 * decltype(jj)::value + 1;
            T r = T(0), i = T(0);
            static_for<H>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                twiddle_acc<((h * k) % G) * (16 / G), T>(v[h], r, i);
            });
            re[k] = r;
            im[k] = i;
        });
    }
};
template <typename T>
struct RealDft<2, T> {
    __device__ __forceinline__ static void run(const T (&x)[2], T (&re)[2], T (&im)[2]) {
        re[0] = x[0] + x[1];
        re[1] = x[0] - x[1];
        (void)im;
    }
};

// Inverse: z holds the spectrum in plane order, already scaled so that
//   y_g = z[0] + (-1)^g z[1] + sum_{0<k<G/2} (z[2k] cos(2pi gk/G) - z[2k+1] sin(2pi gk/G))
// (i.e. 1/G folded into the real planes and 2/G into the complex ones).
// Even/odd split over k: y_g = E_g + O_g, y_{g+G/2} = E_g - O_g.
template <int G, typename T = float>
struct RealIdft {
    static_assert(G >= 4 && (G & (G - 1)) == 0, "G must be a power of two >= 4");
    __device__ __forceinline__ static void run(const T (&z)[G], T (&y)[G]) {
        constexpr int H = G / 2;
        // even frequencies form a length-H spectrum in plane order
        T ze[H];
        ze[0] = z[0];
        ze[1] = z[1];
        static_for<H / 2 - 1>([&](auto jj) {
            constexpr int k2 = decltype(jj)::value + 1;  // sub-frequency k2 <-> k = 2*k2
            ze[2 * k2] = z[4 * k2];
            ze[2 * k2 + 1] = z[4 * k2 + 1];
        });
        T e[H];
        RealIdft<H, T>::run(ze, e);
        static_for<H>([&](auto gg) {
            constexpr int g = decltype(gg)::value;
            T o = T(0);
            static_for<H / 2>([&](auto jj) {
                constexpr int k = 2 * decltype(jj)::value + 1;
                o += rotate_real<((g * k) % G) * (16 / G), T>(z[2 * k], z[2 * k + 1]);
            });
            y[g] = e[g] + o;
            y[g + H] = e[g] - o;
        });
    }
};
template <typename T>
struct RealIdft<2, T> {
    __device__ __forceinline__ static void run(const T (&z)[2], T (&y)[2]) {
        y[0] = z[0] + z[1];
        y[1] = z[0] - z[1];
    }
};

// GELU(v) = v * Phi(v), Phi the standard normal CDF = (1 + erf(v / sqrt 2)) / 2: the
// pointwise nonlinearity of the equivariant MLP block (applied per channel and group
// element, so it commutes with cyclic shifts).
//
// fp32, two values at a time: erf from Abramowitz and Stegun, "Handbook of Mathematical
// Functions", formula 7.1.28 (after Hastings): for x >= 0
//     erf(x) = 1 - (1 + a1 x + a2 x^2 + ... + a6 x^6)^-16 + e(x),   |e(x)| <= 3e-7.
// Written for u = |v| (x = u / sqrt 2): with P(u) = 2^(1/16) (1 + sum_k a_k 2^(-k/2) u^k),
// P(u)^-16 = (1 - erf(u / sqrt 2)) / 2 = Phi(-u), so
//     GELU(v) = max(v, 0) - |v| Phi(-|v|)                  (both signs of v)
// The scale factors are folded into the coefficients, so the cost is six packed FMAs, one
// reciprocal per value (__fdividef, 2 ulp), four packed squarings, one max and one packed
// FMA.  The absolute error stays below 1.3e-6 |v| (7.1e-7 at most), far under the 16-bit
// output rounding.
namespace gelu_coef {
constexpr double kS16 = 1.0442737824274138;   // 2^(1/16)
constexpr double kR2 = 0.70710678118654752;   // 2^(-1/2)
constexpr float c0 = static_cast<float>(kS16);
constexpr float c1 = static_cast<float>(kS16 * 0.0705230784 * kR2);
constexpr float c2 = static_cast<float>(kS16 * 0.0422820123 * kR2 * kR2);
constexpr float c3 = static_cast<float>(kS16 * 0.0092705272 * kR2 * kR2 * kR2);
constexpr float c4 = static_cast<float>(kS16 * 0.0001520143 * kR2 * kR2 * kR2 * kR2);
constexpr float c5 = static_cast<float>(kS16 * 0.0002765672 * kR2 * kR2 * kR2 * kR2 * kR2);
constexpr float c6 = static_cast<float>(kS16 * 0.0000430638 * kR2 * kR2 * kR2 * kR2 * kR2 * kR2);
}  // namespace gelu_coef
__device__ __forceinline__ fx2 gelu2(fx2 v) {
    using namespace gelu_coef;
    const fx2 u(fabsf(v.x), fabsf(v.y));
    fx2 P = fma_t(fx2(c6, c6), u, fx2(c5, c5));
    P = fma_t(P, u, fx2(c4, c4));
    P = fma_t(P, u, fx2(c3, c3));
    P = fma_t(P, u, fx2(c2, c2));
    P = fma_t(P, u, fx2(c1, c1));
    P = fma_t(P, u, fx2(c0, c0));
    fx2 q(__fdividef(1.0f, P.x), __fdividef(1.0f, P.y));   // 1/P underflows to 0 for huge P
    q = q * q;
    q = q * q;
    q = q * q;
    q = q * q;                                              // P^-16 = Phi(-|v|)
    return fma_t(-u, q, fx2(fmaxf(v.x, 0.0f), fmaxf(v.y, 0.0f)));
}
// float64 (the fp32-I/O path): CUDA's erf.
__device__ __forceinline__ double gelu(double v) { return 0.5 * v * (1.0 + erf(v * 0.70710678118654752440)); }

// Epilogue activations (after the bias): 0 = none, 1 = GELU.
constexpr int kActNone = 0;
constexpr int kActGelu = 1;

// Forward transform straight into plane order.
template <int G, typename T>
__device__ __forceinline__ void rdft_planes(const T (&x)[G], T (&p)[G]) {
    T re[G / 2 + 1], im[G / 2 + 1];
    RealDft<G, T>::run(x, re, im);
    p[0] = re[0];
    p[1] = re[G / 2];
#pragma unroll
    for (int k = 1; k < G / 2; ++k) {
        p[2 * k] = re[k];
        p[2 * k + 1] = im[k];
    }
}

}  // namespace eqlin
