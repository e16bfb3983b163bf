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
// cos(pi/4) = sqrt(2)/2, cos(3pi/8) = sqrt(2-sqrt(2))/2, rounded to float.
__host__ __device__ constexpr float cos16(int j) {
    constexpr float c1 = 0.923879532511286756128f;
    constexpr float c2 = 0.707106781186547524401f;
    constexpr float c3 = 0.382683432365089771728f;
    j &= 15;
    switch (j) {
        case 0: return 1.0f;
        case 1: return c1;
        case 2: return c2;
        case 3: return c3;
        case 4: return 0.0f;
        case 5: return -c3;
        case 6: return -c2;
        case 7: return -c1;
        case 8: return -1.0f;
        case 9: return -c1;
        case 10: return -c2;
        case 11: return -c3;
        case 12: return 0.0f;
        case 13: return c3;
        case 14: return c2;
        default: return c1;
    }
}
// sin(2*pi*j/16) = cos(2*pi*(j-4)/16)
__host__ __device__ constexpr float sin16(int j) { return cos16(j - 4); }

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
template <int J>
__device__ __forceinline__ void twiddle_acc(float v, float& re, float& im) {
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
        re = fmaf(v, cos16(j), re);
        im = fmaf(-v, sin16(j), im);
    }
}

// re*cos(2 pi J/16) - im*sin(2 pi J/16), trivial angles without multiplies.
template <int J>
__device__ __forceinline__ float rotate_real(float re, float im) {
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
        return fmaf(re, cos16(j), -im * sin16(j));
    }
}

// Half-spectrum real DFT of length G: x[G] -> re[G/2+1], im[G/2+1]
// (im[0] and im[G/2] are zero and not written).  Decimation in frequency:
// u_h = x_h + x_{h+G/2} carries the even frequencies (a length-G/2 real DFT),
// v_h = x_h - x_{h+G/2} the odd ones.
template <int G>
struct RealDft {
    static_assert(G >= 4 && (G & (G - 1)) == 0, "G must be a power of two >= 4");
    __device__ __forceinline__ static void run(const float (&x)[G], float (&re)[G / 2 + 1],
                                               float (&im)[G / 2 + 1]) {
        constexpr int H = G / 2;
        float u[H], v[H];
#pragma unroll
        for (int h = 0; h < H; ++h) {
            u[h] = x[h] + x[h + H];
            v[h] = x[h] - x[h + H];
        }
        float ure[H / 2 + 1], uim[H / 2 + 1];
        RealDft<H>::run(u, ure, uim);
        static_for<H / 2 + 1>([&](auto kk) {
            constexpr int k = decltype(kk)::value;
            re[2 * k] = ure[k];
            if constexpr (k != 0 && 2 * k != H) im[2 * k] = uim[k];
        });
        // odd frequencies k = 1, 3, ..., H-1
        static_for<H / 2>([&](auto jj) {
            constexpr int k = 2 * decltype(jj)::value + 1;
            float r = 0.0f, i = 0.0f;
            static_for<H>([&](auto hh) {
                constexpr int h = decltype(hh)::value;
                twiddle_acc<((h * k) % G) * (16 / G)>(v[h], r, i);
            });
            re[k] = r;
            im[k] = i;
        });
    }
};
template <>
struct RealDft<2> {
    __device__ __forceinline__ static void run(const float (&x)[2], float (&re)[2], float (&im)[2]) {
        re[0] = x[0] + x[1];
        re[1] = x[0] - x[1];
        (void)im;
    }
};

// Inverse: z holds the spectrum in plane order, already scaled so that
//   y_g = z[0] + (-1)^g z[1] + sum_{0<k<G/2} (z[2k] cos(2pi gk/G) - z[2k+1] sin(2pi gk/G))
// (i.e. 1/G folded into the real planes and 2/G into the complex ones).
// Even/odd split over k: y_g = E_g + O_g, y_{g+G/2} = E_g - O_g.
template <int G>
struct RealIdft {
    static_assert(G >= 4 && (G & (G - 1)) == 0, "G must be a power of two >= 4");
    __device__ __forceinline__ static void run(const float (&z)[G], float (&y)[G]) {
        constexpr int H = G / 2;
        // even frequencies form a length-H spectrum in plane order
        float ze[H];
        ze[0] = z[0];
        ze[1] = z[1];
        static_for<H / 2 - 1>([&](auto jj) {
            constexpr int k2 = decltype(jj)::value + 1;  // sub-frequency k2 <-> k = 2*k2
            ze[2 * k2] = z[4 * k2];
            ze[2 * k2 + 1] = z[4 * k2 + 1];
        });
        float e[H];
        RealIdft<H>::run(ze, e);
        static_for<H>([&](auto gg) {
            constexpr int g = decltype(gg)::value;
            float o = 0.0f;
            static_for<H / 2>([&](auto jj) {
                constexpr int k = 2 * decltype(jj)::value + 1;
                o += rotate_real<((g * k) % G) * (16 / G)>(z[2 * k], z[2 * k + 1]);
            });
            y[g] = e[g] + o;
            y[g + H] = e[g] - o;
        });
    }
};
template <>
struct RealIdft<2> {
    __device__ __forceinline__ static void run(const float (&z)[2], float (&y)[2]) {
        y[0] = z[0] + z[1];
        y[1] = z[0] - z[1];
    }
};

// Forward transform straight into plane order.
template <int G>
__device__ __forceinline__ void rdft_planes(const float (&x)[G], float (&p)[G]) {
    float re[G / 2 + 1], im[G / 2 + 1];
    RealDft<G>::run(x, re, im);
    p[0] = re[0];
    p[1] = re[G / 2];
#pragma unroll
    for (int k = 1; k < G / 2; ++k) {
        p[2 * k] = re[k];
        p[2 * k + 1] = im[k];
    }
}

}  // namespace eqlin
