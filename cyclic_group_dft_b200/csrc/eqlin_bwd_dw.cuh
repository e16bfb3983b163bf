// eqlin_bwd_dw.cuh -- weight and bias gradients of EQ-Linear (16-bit I/O) on sm_100a.
//
// The page "Flash EQ-Linear: Accelerating Equivariant Linear Layers via Group-wise
// Discrete Fourier Transform" lists a backward pass among its kernels (section
// "Implementacion").  For y[n,o,g] = bias[o] + sum_{i,h} w[o,i,(g-h) mod G] x[n,i,h]
// and an upstream gradient dy, the chain rule gives
//     dw[o,i,m] = sum_n sum_g dy[n,o,g] x[n,i,(g-m) mod G]     (a circular
//                 cross-correlation along the group axis, summed over tokens)
//     dbias[o]  = sum_n sum_g dy[n,o,g].
// By the convolution theorem (section "Enfoque Algoritmico") the correlation is a
// pointwise product of spectra, and with real data only the half spectrum is needed:
//     dW_k[o,i] = sum_n DY_k[n,o] conj(X_k[n,i]),   k = 0 .. G/2,
//     dw[o,i,:] = inverse real DFT of dW[o,i,:] (scale 1/G).
// The sum over tokens is a GEMM with K = tokens: per frequency a [Cout x N] by [N x Cin]
// product, 2G-2 real products per K step (4 per complex frequency, 1 per real one).
//
// Kernel eqlin_dw_tc_kernel<G>: the grid is units x token splits.  A unit is an
// (MO-row output tile, NI-column input tile) pair; each CTA owns one unit and a
// contiguous range of 32-token chunks, and keeps its partial dW in TMEM:
//   warp 0      TMA producer: per chunk the dy tile [kTok tokens x MO*G] and the x tile
//               [kTok tokens x NI*G] into a raw ring of p.raw_stages stages (zero fill past
//               N, Cout, Cin), as boxes of kTok rows x kRowBytes (128 B, SWIZZLE_128B; 64 B,
//               SWIZZLE_64B at G = 2).
//   warp 1      MMA issuer + TMEM owner: per chunk and 16-token K step, tcgen05.mma with
//               A = DY^ plane [128 rows (MO valid) x 16 tokens], B = X^ plane [NI x 16],
//               both MN-major (channels contiguous, tokens along K), D plane in TMEM
//               (lane = o, column = i):
//                 D_0 += DY_0 X_0, D_1 += DY_{G/2} X_{G/2},
//                 Re: D_2k   += DYr Xr + DYi Xi,   Im: D_2k+1 += DYi Xr - DYr Xi
//               (the minus through the descriptor's negate-A bit).
//   warps 2..   DFT (dw::Cfg<G>::kDftWarps warps): a unit of work is one token x a few
//               consecutive channels; the 8 lanes of each 16-byte load pass take one
//               channel group of 8 consecutive tokens, which the swizzled boxes spread
//               over 8 bank groups (dw::unit_token); a thread first loads all of its units of a pass, then
//               runs the real DFT over G in fp32 registers (channel pairs packed as fx2),
//               packs each plane to the I/O type and writes one store per plane into the
//               MN-major SWIZZLE_64B spectra.  The dy units also add plane 0 (the group
//               sum) to a per-token slot for dbias, each slot with a single writer, so the
//               sums are formed in a fixed order.  Spectra use p.spec_bufs buffers.
//               After the last chunk the same warps read the TMEM partial dW and write it
//               to the CTA's slab of the workspace.
// eqlin_dw_finish_kernel<G> then sums the slabs of each unit over its token splits in a
// fixed order (deterministic, float64), runs the inverse real DFT over the planes in
// float64 and writes dw (fp32) and dbias (fp32).
//
// Spectra layout (one buffer): A = G planes of 4 K-groups x MA atoms of 512 bytes
// (MA = ceil(MO / 32)), then slack: a 128-row MMA reads 4 atoms along M, so for MO < 128
// it reads into the next K group (or the slack after the last plane); those D rows are
// never read back.  B = G planes of 4 x NA atoms (NA = ceil(NI / 32)).
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "eqlin_layout.h"
#include "group_dft.cuh"
#include "io16.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

struct DwParams {
    float* ws;                 // workspace: per CTA a slab [G][NI][MO] fp32 followed by [MO] bias sums
    int* status;               // device status word (first error wins)
    long long N;
    int MO, NI;                // rows / columns of a unit (multiples of 16; MO <= 128, G*NI <= 512)
    int n_it;                  // input tiles per output tile
    int n_splits;              // CTAs per unit (token splits)
    long long n_chunks;        // ceil(N / kTok)
    int cpb_dy, cpb_x;         // channels per TMA box of the dy / x tile
    uint32_t dy_bytes;         // dy part of a raw stage: kTok * MO * G * 2
    uint32_t raw_bytes;        // one raw stage: dy part + x part (multiple of 1 KB)
    uint32_t a_bytes;          // A (dy spectra) region of one spectra buffer (multiple of 1 KB)
    uint32_t b_bytes;          // B (x spectra) region (multiple of 1 KB)
    uint32_t tmem_cols;        // power of two >= G * NI
    int raw_stages;            // depth of the raw ring (2 .. kMaxRawStages)
    int spec_bufs;             // spectra buffers (1 or 2)
    int MA, NA;                // 32-channel atoms per plane row group: ceil(MO / 32), ceil(NI / 32)
    size_t slab_floats;        // G * NI * MO (a CTA's slab holds slab_floats + MO floats)
    unsigned long long timeout_ns;
};

namespace dw {

constexpr int kMaxRawStages = 8;   // raw ring depth is a launch parameter (p.raw_stages)
constexpr int kMaxSpecBufs = 2;
constexpr int kWarpProducer = 0;
constexpr int kWarpMma = 1;
constexpr int kWarpDft0 = 2;

// Transform warps per CTA: 16 (4 per SM sub-partition, to hide the latency of the short
// dependent DFT chains); with the per-token units the transform needs <= 112 registers.
template <int G>
struct Cfg {
    // tokens per chunk: 32 (two MMA K steps) for G <= 4; 16 for G >= 8, where a token's
    // raw rows are twice as long, so that the raw ring keeps four or more stages (B200:
    // weight gradient of C16 C32 218 vs 258 us, p8 C64 30.8 vs 35.0 us; p4 C96 81.4 us with
    // 32 tokens against 98.4 with 16)
    static constexpr int kTok = G >= 8 ? 16 : 32;
    static constexpr int kKGroups = kTok / 8;   // 8-token K groups per spectra plane
    static constexpr int kDftWarps = 16;
    static constexpr int kDftThreads = kDftWarps * 32;
    static constexpr int kThreads = (2 + kDftWarps) * 32;
    // channels per transform unit: one 16-byte store per plane for G <= 4, 8 bytes for
    // G = 8, 4 bytes for G = 16 (where the DFT itself dominates and threads are plenty)
    static constexpr int kChanPerUnit = G <= 4 ? 8 : (G == 8 ? 4 : 2);
    // units per transform thread and chunk, at most: kTok tokens x (MO + NI) / kChanPerUnit
    // with MO <= 128 and G * NI <= 512, NI <= 256
    static constexpr int kMaxUnits = kTok * (128 + (512 / G < 256 ? 512 / G : 256)) / kChanPerUnit;
    static constexpr int kMaxPasses = (kMaxUnits + kDftThreads - 1) / kDftThreads;
    // raw box rows: 128 B (SWIZZLE_128B) of kBoxChannels channels x G, 64 B (SWIZZLE_64B)
    // at G = 2; a unit (kChanPerUnit channels, 32 or 64 bytes) never straddles two boxes
    static constexpr int kRowBytes = G == 2 ? 64 : 128;
    static constexpr int kBoxChannels = kRowBytes / (2 * G);
    static_assert(kBoxChannels % kChanPerUnit == 0, "units inside boxes");

};
constexpr int kBarDft = 1;         // named barrier among the DFT warps
constexpr uint32_t kWaitSleepNs = 20000;

struct Ctl {
    volatile int abort;
    uint32_t tmem_base;
};

// Bounded mbarrier wait; false (after flagging) on timeout or abort.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, Ctl* ctl, int* status,
                                             unsigned long long timeout_ns) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (ptx::mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if ((spin & 7u) == 0) {
            if (ctl->abort) return false;
            if (ptx::globaltimer_ns() - t0 > timeout_ns) {
                ctl->abort = 1;
                atomicCAS(status, 0, kDeviceErrTimeout);
                return false;
            }
        }
    }
}

// Wait that ignores the abort flag (for copies or MMAs in flight before exit).
__device__ __forceinline__ void drain_wait(uint32_t bar, uint32_t parity, int* status,
                                           unsigned long long timeout_ns) {
    const uint64_t t0 = ptx::globaltimer_ns();
    while (!ptx::mbar_try_wait(bar, parity)) {
        if (ptx::globaltimer_ns() - t0 > timeout_ns) {
            atomicCAS(status, 0, kDeviceErrTimeout);
            return;
        }
    }
}


// One unit of the transform: one token t of the chunk x CPU consecutive channels
// c0 .. c0+CPU-1 of the dy tile or of the x tile (CPU = Cfg<G>::kChanPerUnit).  `row` is
// the token's row of the box holding the unit; the unit's k-th 16-byte piece is logical
// piece lc + k of the row, stored at piece (lc + k) ^ key (key = t % 8 for 128-byte
// SWIZZLE_128B rows, (t / 2) % 4 for 64-byte SWIZZLE_64B rows).  The unit's CPU*G values
// are CPU*G/2 32-bit words, channel c0+j in words j*G/2 .. (j+1)*G/2-1.
template <int G, int CPU>
__device__ __forceinline__ void load_unit(const uint8_t* row, int lc, int key, uint32_t (&w)[CPU * G / 2]) {
    constexpr int BYTES = CPU * G * 2;
    constexpr int PIECES = BYTES / 16;       // 2 or 4 sixteen-byte pieces
    static_assert(BYTES == 32 || BYTES == 64, "unit size");
#pragma unroll
    for (int k = 0; k < PIECES; ++k) {
        const uint4 v = *reinterpret_cast<const uint4*>(row + 16 * ((lc + k) ^ key));
        w[4 * k + 0] = v.x;
        w[4 * k + 1] = v.y;
        w[4 * k + 2] = v.z;
        w[4 * k + 3] = v.w;
    }
}

// Token and channel group of unit v of a tile with ng groups of CPU channels per token:
// v = ((token / 8) * ng + group) * 8 + token % 8, so consecutive lanes take 8 consecutive
// tokens of one group, then the next group.
__device__ __forceinline__ void unit_token(int v, int ng, int& tok, int& grp) {
    const int rest = v >> 3;
    grp = rest % ng;
    tok = (rest / ng) * 8 + (v & 7);
}

// Real DFT over G of the unit's channels (in pairs packed as fx2), stored to the planes in
// the MN-major SWIZZLE_64B operand layout: plane p of the unit at dst + p * plane_bytes
// (dst from unit_dst_offset).  One store of CPU * 2 bytes per plane.  With with_bias,
// adds plane 0 (the group sums) to the thread's running dbias sums bias[0..CPU) (kept in
// registers across chunks).
template <int G, int CPU, class T16>
__device__ __forceinline__ void store_unit(const uint32_t (&w)[CPU * G / 2], uint8_t* dst, uint32_t plane_bytes,
                                           float (&bias)[CPU], bool with_bias) {
    constexpr int H = G / 2;
    uint32_t packed[G][CPU / 2];
#pragma unroll
    for (int j = 0; j < CPU / 2; ++j) {      // channels c0 + 2j, c0 + 2j + 1
        fx2 v[G], pl[G];
#pragma unroll
        for (int h = 0; h < H; ++h) {
            const uint32_t a = w[(2 * j) * H + h], b = w[(2 * j + 1) * H + h];
            v[2 * h] = fx2(Io16<T16>::lo(a), Io16<T16>::lo(b));
            v[2 * h + 1] = fx2(Io16<T16>::hi(a), Io16<T16>::hi(b));
        }
        rdft_planes<G>(v, pl);
        if (with_bias) {
            bias[2 * j] += pl[0].x;
            bias[2 * j + 1] += pl[0].y;
        }
#pragma unroll
        for (int p = 0; p < G; ++p) packed[p][j] = Io16<T16>::pack(pl[p].x, pl[p].y);
    }
#pragma unroll
    for (int p = 0; p < G; ++p) {
        uint8_t* d = dst + p * plane_bytes;
        if constexpr (CPU == 8) {
            *reinterpret_cast<uint4*>(d) = make_uint4(packed[p][0], packed[p][1], packed[p][2], packed[p][3]);
        } else if constexpr (CPU == 4) {
            *reinterpret_cast<uint2*>(d) = make_uint2(packed[p][0], packed[p][1]);
        } else {
            *reinterpret_cast<uint32_t*>(d) = packed[p][0];
        }
    }
}

// Offset of channel c0 of token t in a plane of the MN-major SWIZZLE_64B layout: the 8-row
// atom (kg = t / 8, ma = c0 / 32) at kg * sbo + ma * 512 holds row t % 8 = 64 bytes of
// channels 32ma .. 32ma + 31, 16-byte chunk j of row r stored at chunk j ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t unit_dst_offset(int t, int c0, uint32_t sbo) {
    const int r = t & 7;
    return static_cast<uint32_t>(t >> 3) * sbo + static_cast<uint32_t>(c0 >> 5) * 512u + static_cast<uint32_t>(r) * 64u +
           static_cast<uint32_t>((((c0 & 31) >> 3) ^ ((r >> 1) & 3)) << 4) + static_cast<uint32_t>(c0 & 7) * 2u;
}

}  // namespace dw

template <int G, class T16>
__global__ void __launch_bounds__(dw::Cfg<G>::kThreads, 1)
    eqlin_dw_tc_kernel(const __grid_constant__ CUtensorMap tmap_dy, const __grid_constant__ CUtensorMap tmap_x,
                       const DwParams p) {
    constexpr int kDftThreads = dw::Cfg<G>::kDftThreads;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* base = ptx::smem_align_1k(smem_raw);
    const uint32_t spec_bytes = p.a_bytes + p.b_bytes;
    uint8_t* raw0 = base;
    uint8_t* spec0 = raw0 + p.raw_stages * p.raw_bytes;
    float* bias_sm = reinterpret_cast<float*>(spec0 + p.spec_bufs * spec_bytes);
    // bias_sm[t][c]: group sums of dy channel c at chunk token t, over every chunk; each
    // slot has a single writer (the unit -> thread map is the same for every chunk), so
    // the per-CTA sums are formed in a fixed order
    uint64_t* bars = reinterpret_cast<uint64_t*>(bias_sm + dw::Cfg<G>::kTok * p.MO);
    const int RS = p.raw_stages, SB = p.spec_bufs;
    dw::Ctl* ctl = reinterpret_cast<dw::Ctl*>(bars + 2 * RS + 2 * SB + 2);

    auto bar_raw_full = [&](int s) { return ptx::smem_u32(bars + s); };
    auto bar_raw_empty = [&](int s) { return ptx::smem_u32(bars + RS + s); };
    auto bar_spec_full = [&](int s) { return ptx::smem_u32(bars + 2 * RS + s); };
    auto bar_spec_empty = [&](int s) { return ptx::smem_u32(bars + 2 * RS + SB + s); };
    const uint32_t bar_acc_full = ptx::smem_u32(bars + 2 * RS + 2 * SB);
    const uint32_t bar_drain = ptx::smem_u32(bars + 2 * RS + 2 * SB + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int unit = blockIdx.x / p.n_splits, split = blockIdx.x - unit * p.n_splits;
    const int ot = unit / p.n_it, it = unit - ot * p.n_it;
    const int o0 = ot * p.MO, i0 = it * p.NI;
    const long long c_begin = p.n_chunks * split / p.n_splits;
    const long long c_end = p.n_chunks * (split + 1) / p.n_splits;
    const int n_mine = static_cast<int>(c_end - c_begin);

    if (threadIdx.x == 0) {
        for (int s = 0; s < RS; ++s) {
            ptx::mbar_init(bar_raw_full(s), 1);
            ptx::mbar_init(bar_raw_empty(s), kDftThreads);
        }
        for (int s = 0; s < SB; ++s) {
            ptx::mbar_init(bar_spec_full(s), kDftThreads);
            ptx::mbar_init(bar_spec_empty(s), 1);
        }
        ptx::mbar_init(bar_acc_full, 1);
        ptx::mbar_init(bar_drain, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == dw::kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), p.tmem_cols);
        ptx::tmem_relinquish();
    }
    if (warp == dw::kWarpProducer && lane == 0) {
        ptx::prefetch_tmap(&tmap_dy);
        ptx::prefetch_tmap(&tmap_x);
    }
    if (warp >= dw::kWarpDft0) {
        const int t = threadIdx.x - dw::kWarpDft0 * 32;

        // A-region tail rows (read by the MMA, never written by the transform): zero
        // A-region slack after the G planes (read by the 128-row MMA of the last plane,
        // never written by the transform): zero
        const uint32_t tail0 = static_cast<uint32_t>(G) * dw::Cfg<G>::kKGroups * static_cast<uint32_t>(p.MA) * 512u;
        for (int b = 0; b < SB; ++b) {
            uint8_t* a = spec0 + static_cast<size_t>(b) * spec_bytes;
            for (uint32_t idx = tail0 / 16 + t; idx < p.a_bytes / 16; idx += kDftThreads)
                reinterpret_cast<uint4*>(a)[idx] = make_uint4(0, 0, 0, 0);
        }
        ptx::fence_proxy_async_smem();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();

    if (warp == dw::kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            const int nb_dy = p.MO / p.cpb_dy, nb_x = p.NI / p.cpb_x;
            const uint32_t box_dy = dw::Cfg<G>::kTok * p.cpb_dy * G * 2, box_x = dw::Cfg<G>::kTok * p.cpb_x * G * 2;
            const uint32_t tx = p.dy_bytes + dw::Cfg<G>::kTok * p.NI * G * 2;
            const uint32_t s_raw0 = ptx::smem_u32(raw0);
            int issued = 0;
            for (int j = 0; j < n_mine; ++j) {
                const int s = j % RS;
                const uint32_t ph = static_cast<uint32_t>(j / RS) & 1u;
                if (!dw::wait_bounded(bar_raw_empty(s), ph ^ 1u, ctl, p.status, p.timeout_ns)) break;
                const int n0 = static_cast<int>((c_begin + j) * dw::Cfg<G>::kTok);
                const uint32_t dst = s_raw0 + s * p.raw_bytes;
                ptx::mbar_arrive_expect_tx(bar_raw_full(s), tx);
                for (int b = 0; b < nb_dy; ++b)
                    ptx::tma_load_2d(dst + b * box_dy, &tmap_dy, (o0 + b * p.cpb_dy) * G, n0, bar_raw_full(s));
                for (int b = 0; b < nb_x; ++b)
                    ptx::tma_load_2d(dst + p.dy_bytes + b * box_x, &tmap_x, (i0 + b * p.cpb_x) * G, n0,
                                     bar_raw_full(s));
                ++issued;
            }
            // every copy issued must land before the CTA exits
            for (int s = 0; s < RS && s < issued; ++s) {
                const int last = ((issued - 1 - s) / RS) * RS + s;
                dw::drain_wait(bar_raw_full(s), static_cast<uint32_t>(last / RS) & 1u, p.status,
                               p.timeout_ns);
            }
        }
    } else if (warp == dw::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // both operands MN-major (channels contiguous, tokens along K)
            const uint32_t ID = idesc_f16kind_f32_mn(kMmaM, p.NI, Io16<T16>::kUmmaFormat, false);
            const uint32_t ID_NEG = idesc_f16kind_f32_mn(kMmaM, p.NI, Io16<T16>::kUmmaFormat, true);
            const uint32_t s_spec0 = ptx::smem_u32(spec0);
            const uint32_t sbo_a = static_cast<uint32_t>(p.MA) * 512u, sbo_b = static_cast<uint32_t>(p.NA) * 512u;
            const uint32_t hi_a = ptx::sdesc_mn_sw64_hi(sbo_a), hi_b = ptx::sdesc_mn_sw64_hi(sbo_b);
            const uint32_t plane_a16 = dw::Cfg<G>::kKGroups * sbo_a / 16u, plane_b16 = dw::Cfg<G>::kKGroups * sbo_b / 16u;
            bool ok = true;
            for (int j = 0; j < n_mine; ++j) {
                const int sb = j % SB;
                const uint32_t ph = static_cast<uint32_t>(j / SB) & 1u;
                if (!dw::wait_bounded(bar_spec_full(sb), ph, ctl, p.status, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t a_addr = s_spec0 + sb * spec_bytes;
                const uint32_t a_lo = ptx::sdesc_mn_sw64_lo(a_addr, 512u);
                const uint32_t b_lo = ptx::sdesc_mn_sw64_lo(a_addr + p.a_bytes, 512u);
#pragma unroll
                for (int ks = 0; ks < dw::Cfg<G>::kTok / 16; ++ks) {
                    const uint32_t acc0 = (j > 0 || ks > 0) ? 1u : 0u;
                    // K step ks = tokens 16ks .. 16ks+15 = K groups 2ks, 2ks+1
                    auto A = [&](int pl) {
                        return ptx::sdesc_from_halves(hi_a, a_lo + pl * plane_a16 + 2 * ks * (sbo_a / 16));
                    };
                    auto B = [&](int pl) {
                        return ptx::sdesc_from_halves(hi_b, b_lo + pl * plane_b16 + 2 * ks * (sbo_b / 16));
                    };
                    auto D = [&](int pl) { return tmem_base + static_cast<uint32_t>(pl * p.NI); };
                    ptx::umma_f16(D(0), A(0), B(0), ID, acc0);
                    ptx::umma_f16(D(1), A(1), B(1), ID, acc0);
#pragma unroll
                    for (int k = 1; k < G / 2; ++k) {
                        const int pr = 2 * k, pi = 2 * k + 1;
                        ptx::umma_f16(D(pr), A(pr), B(pr), ID, acc0);      // + DYr Xr
                        ptx::umma_f16(D(pr), A(pi), B(pi), ID, 1u);        // + DYi Xi
                        ptx::umma_f16(D(pi), A(pi), B(pr), ID, acc0);      // + DYi Xr
                        ptx::umma_f16(D(pi), A(pr), B(pi), ID_NEG, 1u);    // - DYr Xi
                    }
                }
                ptx::umma_commit(bar_spec_empty(sb));
            }
            if (ok) ptx::umma_commit(bar_acc_full);
            ptx::umma_commit(bar_drain);
            dw::drain_wait(bar_drain, 0, p.status, p.timeout_ns);
        }
    } else {
        // ------------------------------------------------------------ transform warps
        const int t = threadIdx.x - dw::kWarpDft0 * 32;
        // units: token t x CPU channels; the dy units of all tokens first, then x's.  A
        // thread handles units t + ps * kDftThreads, the same ones in every chunk, so it
        // keeps the dbias sums of its dy units in registers (bsum) until the end.
        constexpr int CPU = dw::Cfg<G>::kChanPerUnit;
        const int groups_dy = p.MO / CPU, groups_x = p.NI / CPU;
        const int units_dy = dw::Cfg<G>::kTok * groups_dy;
        const int n_units = units_dy + dw::Cfg<G>::kTok * groups_x;
        float bsum[dw::Cfg<G>::kMaxPasses][CPU];
#pragma unroll
        for (int ps = 0; ps < dw::Cfg<G>::kMaxPasses; ++ps)
#pragma unroll
            for (int j = 0; j < CPU; ++j) bsum[ps][j] = 0.0f;
        const uint32_t sbo_a = static_cast<uint32_t>(p.MA) * 512u, sbo_b = static_cast<uint32_t>(p.NA) * 512u;
        const uint32_t plane_a = dw::Cfg<G>::kKGroups * sbo_a, plane_b = dw::Cfg<G>::kKGroups * sbo_b;
        // the thread's units are the same in every chunk: their source offsets in a raw
        // stage and destination offsets in a spectra buffer are computed once
        constexpr int MP = dw::Cfg<G>::kMaxPasses;
        uint32_t src_off[MP], dst_off[MP];
        uint8_t lc_key[MP];
        uint32_t dy_mask = 0, valid_mask = 0;
#pragma unroll
        for (int ps = 0; ps < MP; ++ps) {
            const int u = t + ps * kDftThreads;
            src_off[ps] = dst_off[ps] = 0;
            lc_key[ps] = 0;
            if (u < n_units) {
                const bool is_dy = u < units_dy;
                const int v = is_dy ? u : u - units_dy, ng = is_dy ? groups_dy : groups_x;
                int tok, grp;
                dw::unit_token(v, ng, tok, grp);
                const int c = CPU * grp;
                constexpr int RB = dw::Cfg<G>::kRowBytes, CPB = dw::Cfg<G>::kBoxChannels;
                const int box = c / CPB;
                src_off[ps] = (is_dy ? 0u : p.dy_bytes) + static_cast<uint32_t>(box * (dw::Cfg<G>::kTok * RB) + tok * RB);
                const int lc = (c - box * CPB) * G * 2 / 16;
                const int key = RB == 128 ? (tok & 7) : ((tok >> 1) & 3);
                lc_key[ps] = static_cast<uint8_t>(lc | (key << 4));
                dst_off[ps] = (is_dy ? 0u : p.a_bytes) + dw::unit_dst_offset(tok, c, is_dy ? sbo_a : sbo_b);
                valid_mask |= 1u << ps;
                if (is_dy) dy_mask |= 1u << ps;
            }
        }
        bool ok = true;
        for (int j = 0; j < n_mine; ++j) {
            const int s = j % RS, sb = j % SB;
            const uint32_t ph_raw = static_cast<uint32_t>(j / RS) & 1u;
            const uint32_t ph_spec = static_cast<uint32_t>(j / SB) & 1u;
            // no barrier among the transform warps: each thread waits for itself, and a
            // timeout (which sets the abort flag for every role) ends the loop for all
            if (!dw::wait_bounded(bar_raw_full(s), ph_raw, ctl, p.status, p.timeout_ns) ||
                !dw::wait_bounded(bar_spec_empty(sb), ph_spec ^ 1u, ctl, p.status, p.timeout_ns)) {
                ok = false;
                break;
            }
            const uint8_t* raw = raw0 + static_cast<size_t>(s) * p.raw_bytes;
            uint8_t* spec = spec0 + static_cast<size_t>(sb) * spec_bytes;
#pragma unroll
            for (int ps = 0; ps < MP; ++ps) {
                if (!(valid_mask & (1u << ps))) break;
                uint32_t words[CPU * G / 2];
                dw::load_unit<G, CPU>(raw + src_off[ps], lc_key[ps] & 15, lc_key[ps] >> 4, words);
                const bool is_dy = dy_mask & (1u << ps);
                dw::store_unit<G, CPU, T16>(words, spec + dst_off[ps], is_dy ? plane_a : plane_b, bsum[ps], is_dy);
            }
            ptx::fence_proxy_async_smem();
            ptx::mbar_arrive(bar_raw_empty(s));
            ptx::mbar_arrive(bar_spec_full(sb));
        }
        // partial dW: TMEM -> this CTA's workspace slab [G][NI][MO]
        const bool got = ok && dw::wait_bounded(bar_acc_full, 0, ctl, p.status, p.timeout_ns);
        const bool all = ptx::named_bar_and(dw::kBarDft, kDftThreads, got);
        float* slab = p.ws + static_cast<size_t>(blockIdx.x) * (p.slab_floats + p.MO);
        if (all) {
            ptx::tc_fence_after();
            // the warps of lane quarter q (warp % 4) share its planes round-robin
            constexpr int kGroups = dw::Cfg<G>::kDftWarps / 4;
            const int q = warp & 3, grp = (warp - dw::kWarpDft0) >> 2;
            const int row = q * 32 + lane;
            if (q * 32 < p.MO) {
                for (int pl = grp; pl < G; pl += kGroups) {
                    for (int cb = 0; cb < p.NI; cb += 16) {
                        uint32_t v[16];
                        ptx::tmem_ld_32x32b<16>(tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                                    static_cast<uint32_t>(pl * p.NI + cb),
                                                v);
                        ptx::tmem_wait_ld();
                        if (row < p.MO) {
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                slab[(static_cast<size_t>(pl) * p.NI + cb + e) * p.MO + row] = __uint_as_float(v[e]);
                        }
                    }
                }
            }
        }
        // dbias partial of this CTA (every CTA writes it; the inverse-DFT kernel reads input
        // tile 0's): each thread's register sums to their slots bias_sm[tok][c], then per
        // channel the kTok token slots in order
#pragma unroll
        for (int ps = 0; ps < dw::Cfg<G>::kMaxPasses; ++ps) {
            const int u = t + ps * kDftThreads;
            if (u < units_dy) {
                int tok, grp;
                dw::unit_token(u, groups_dy, tok, grp);
                const int c = CPU * grp;
#pragma unroll
                for (int j = 0; j < CPU; ++j) bias_sm[tok * p.MO + c + j] = bsum[ps][j];
            }
        }
        ptx::named_bar_sync(dw::kBarDft, kDftThreads);
        for (int c = t; c < p.MO; c += kDftThreads) {
            float acc = 0.0f;
            for (int tok = 0; tok < dw::Cfg<G>::kTok; ++tok) acc += bias_sm[tok * p.MO + c];
            slab[p.slab_floats + c] = acc;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == dw::kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, p.tmem_cols);
    }
}

// Cross-CTA reduction and inverse DFT, deterministic, in one small kernel.
// Block = (unit u, column ii of the unit, 32 consecutive rows oo), or the unit's bias
// sums when ii == NI.  Warp w of the block's W warps sums the slabs of splits w, w+W,
// w+2W, ... in that order, float64, for the block's G planes, with kIn splits (kIn * G
// loads per thread) in flight per round trip; the W warp sums are then added in warp
// order.  W = 16: 148 splits then take one round trip per warp, not three.  The W x G x 32
// float64 warp sums live in dynamic shared memory (64 KB at G = 16).  Launched as a
// programmatic dependent of the main kernel: its blocks start as that kernel's CTAs
// exit and wait (griddepcontrol.wait) for all of its slabs before reading them.
// With P_k = sum_n DY_k conj(X_k) (unscaled transforms), warp 0 writes
//   dw[o,i,m] = (1/G) [P_0 + (-1)^m P_{G/2} + 2 sum_{0<k<G/2} Re(P_k e^{+2 pi i m k / G})],
// and dbias[o] from the bias sums of the units of input tile 0.
struct DwFinalParams {
    const float* ws;      // slabs: per CTA [G][NI][MO] then [MO]
    float* dw;            // [Cout, Cin, G]
    float* dbias;         // [Cout] or nullptr
    int Cout, Cin;
    int MO, NI, n_it, n_splits;
    size_t slab_floats;   // G * NI * MO
};

constexpr int kDwFinishWarps = 16;

template <int G>
__global__ void __launch_bounds__(kDwFinishWarps * 32) eqlin_dw_finish_kernel(const DwFinalParams f) {
    constexpr int W = kDwFinishWarps;
    extern __shared__ double red_sm[];   // [W][G][32]
    auto red = [&](int w, int pl) -> double& { return red_sm[(w * G + pl) * 32 + (threadIdx.x & 31)]; };
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();
    const int n_og = (f.MO + 31) / 32;
    const int per_unit = (f.NI + 1) * n_og;
    const int unit = static_cast<int>(blockIdx.x) / per_unit;
    const int rem = static_cast<int>(blockIdx.x) % per_unit;
    const int ii = rem / n_og, oo = (rem % n_og) * 32 + (threadIdx.x & 31);
    const int warp = threadIdx.x >> 5;
    const bool bias_blk = ii == f.NI;
    const size_t stride = f.slab_floats + f.MO;
    const size_t pstride = static_cast<size_t>(f.NI) * f.MO;   // between planes of a slab
    double acc[G];
#pragma unroll
    for (int pl = 0; pl < G; ++pl) acc[pl] = 0.0;
    if (oo < f.MO) {
        const float* src = f.ws + static_cast<size_t>(unit) * f.n_splits * stride +
                           (bias_blk ? f.slab_floats + oo : static_cast<size_t>(ii) * f.MO + oo);
        const int nv = bias_blk ? 1 : G;
        int s = warp;
        // kIn splits in flight per round trip, added in split order.  Measured on B200
        // (weight gradient, reduction included): G = 4 with 8 (64 registers, two blocks per
        // SM) 71.0 us at p4 C96, with 10 (76 registers) 73.3; G = 8 with 8 (122 registers)
        // 26.4 us at p8 C64, with 4 30.7; G = 16 with 4 (128 registers) 176.1 us at C16,
        // with 2 (and the spills of a fully unrolled warp sum) 177.7
        constexpr int kIn = G <= 4 ? 32 / G : (G == 8 ? 8 : 4);
        for (; s + W * (kIn - 1) < f.n_splits; s += W * kIn) {
            float v[kIn][G];
#pragma unroll
            for (int u = 0; u < kIn; ++u) {
#pragma unroll
                for (int pl = 0; pl < G; ++pl)
                    if (pl < nv) v[u][pl] = src[static_cast<size_t>(s + W * u) * stride + pl * pstride];
            }
#pragma unroll
            for (int u = 0; u < kIn; ++u) {
#pragma unroll
                for (int pl = 0; pl < G; ++pl)
                    if (pl < nv) acc[pl] += v[u][pl];
            }
        }
        for (; s < f.n_splits; s += W) {
#pragma unroll
            for (int pl = 0; pl < G; ++pl)
                if (pl < nv) acc[pl] += src[static_cast<size_t>(s) * stride + pl * pstride];
        }
    }
#pragma unroll
    for (int pl = 0; pl < G; ++pl) red(warp, pl) = acc[pl];
    __syncthreads();
    if (warp != 0 || oo >= f.MO) return;
    double z[G];
    // fully unrolled, the warp sum's G x W shared loads spill at G >= 8 (512 and 1564 B)
    constexpr int kSumUnroll = G <= 4 ? W : 4;
#pragma unroll
    for (int pl = 0; pl < G; ++pl) {
        double v = 0.0;
#pragma unroll kSumUnroll
        for (int w = 0; w < W; ++w) v += red(w, pl);   // in warp order (deterministic)
        z[pl] = v;
    }
    const int ot = unit / f.n_it, it = unit % f.n_it;
    const int o = ot * f.MO + oo;
    if (o >= f.Cout) return;
    if (bias_blk) {
        if (f.dbias != nullptr && it == 0) f.dbias[o] = static_cast<float>(z[0]);
        return;
    }
    const int i = it * f.NI + ii;
    if (i >= f.Cin) return;
#pragma unroll
    for (int pl = 0; pl < G; ++pl) z[pl] = (pl < 2 ? z[pl] : 2.0 * z[pl]) / G;
    double out[G];
    if constexpr (G == 2) {
        out[0] = z[0] + z[1];
        out[1] = z[0] - z[1];
    } else {
        RealIdft<G, double>::run(z, out);
    }
    float* dst = f.dw + (static_cast<size_t>(o) * f.Cin + i) * G;
#pragma unroll
    for (int m = 0; m < G; ++m) dst[m] = static_cast<float>(out[m]);
}

// ------------------------------------------------------------------ fp32 I/O
// Weight and bias gradients for fp32 I/O on CUDA cores in float64, straight from the
// definition: thread = (o, i) pair, blockIdx.y = token slice; partial sums are added
// to a float64 accumulator [Cout][Cin][G] followed by [Cout] (zeroed by the caller),
// which eqlin_dw_f64_convert_kernel rounds to fp32.
template <int G>
__global__ void __launch_bounds__(256)
    eqlin_dw_f64_kernel(const float* __restrict__ x, const float* __restrict__ dy, double* __restrict__ acc,
                        long long N, int Cin, int Cout, long long tokens_per_slice) {
    const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<long long>(Cout) * Cin) return;
    const int o = static_cast<int>(idx / Cin), i = static_cast<int>(idx % Cin);
    const long long n0 = static_cast<long long>(blockIdx.y) * tokens_per_slice;
    const long long n1 = n0 + tokens_per_slice < N ? n0 + tokens_per_slice : N;
    double s[G], b = 0.0;
#pragma unroll
    for (int m = 0; m < G; ++m) s[m] = 0.0;
    for (long long n = n0; n < n1; ++n) {
        double d[G], xv[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            d[g] = dy[(n * Cout + o) * G + g];
            xv[g] = x[(n * Cin + i) * G + g];
        }
#pragma unroll
        for (int m = 0; m < G; ++m) {
#pragma unroll
            for (int g = 0; g < G; ++g) s[m] = fma(d[g], xv[(g - m + G) % G], s[m]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) b += d[g];
    }
    if (n1 <= n0) return;
#pragma unroll
    for (int m = 0; m < G; ++m) atomicAdd(acc + (static_cast<size_t>(o) * Cin + i) * G + m, s[m]);
    if (i == 0) atomicAdd(acc + static_cast<size_t>(Cout) * Cin * G + o, b);
}

__global__ void eqlin_dw_f64_convert_kernel(const double* __restrict__ acc, float* __restrict__ dw,
                                            float* __restrict__ dbias, size_t n_w, int Cout) {
    const size_t idx = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx < n_w) dw[idx] = static_cast<float>(acc[idx]);
    if (dbias != nullptr && idx < static_cast<size_t>(Cout)) dbias[idx] = static_cast<float>(acc[n_w + idx]);
}

}  // namespace eqlin
