// eqlin_mlp.cuh -- the equivariant MLP block y = L2(GELU(L1(x))) as ONE persistent kernel.
//
// Page "Flash EQ-Linear: Accelerating Equivariant Linear Layers via Group-wise Discrete
// Fourier Transform": the network-level gains (section "A Nivel de Red") come from
// networks whose blocks chain EQ-Linear layers; section "Implementacion" keeps the
// Fourier fragments on chip between the steps.  Here the two layers and the pointwise
// GELU between them run in one kernel and the hidden activation [N, H, G] never leaves
// the SM:
//     X^ = rDFT(x)                                  (per token tile, resident)
//     for each 128-row hidden chunk:
//         Y1^_k = W1^_k X^_k                        (tcgen05, TMEM accumulator acc1)
//         h    = GELU(irDFT(Y1^) + b1)              (epilogue warps, fp32 registers)
//         H^   = rDFT(h)                            (same registers, to shared memory)
//         Y2^_k += W2^_k H^_k                       (tcgen05, TMEM accumulator acc2)
//     y = irDFT(Y2^) + b2                           (epilogue warps, straight to HBM)
// GELU is pointwise in the group domain, so it commutes with the cyclic shift and the
// block stays equivariant.
//
// Tokens are the MMA N dimension, as in eqlin_fwd_tc.cuh: BN = 512 / (2G) tokens per
// tile, acc1 and acc2 G*BN TMEM columns each.  The hidden spectrum H^ of one hidden chunk
// is written in the same K-major SWIZZLE_64B pair-slot layout as X^ ([-Im, Re, Im] per
// complex frequency, eqlin_layout.h), so both products are issued exactly like the
// single layer's.  Weights stream from L2 in units of one frequency (two planes of a
// 128-row x 32-channel chunk, 16 KB) through a ring, in the order the MMAs use them.
//
// Roles per CTA (one per SM, persistent over token tiles):
//   warp 12     producer: x chunks of a tile (TMA) into resident slots, weight units into
//               the ring (bulk copies)
//   warps 8-11  DFT of each x chunk in place (tc::dft_chunk), then a third of each hidden
//               chunk's epilogue with the epilogue warps
//   warp 13     MMA issuer + TMEM owner.  Per tile: for each hidden chunk hc, the layer-1
//               products into acc1, then (once the epilogue has written H^ of hc-1) the
//               layer-2 products of hc-1 into acc2
//   warps 0-7   epilogue: two thirds of each hidden chunk (acc1 -> H^) and, per tile, the
//               output (acc2 -> y)
// Waits are bounded as in eqlin_fwd_tc.cuh.
#pragma once

#include <cstdint>

#include "eqlin_fwd_tc.cuh"
#include "eqlin_layout.h"
#include "eqlin_prep.cuh"
#include "group_dft.cuh"
#include "io16.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

struct MlpParams {
    const uint8_t* w1_img;   // W1^ image [hc][c][p][r < 128][32] (eqlin_layout.h), H rows in 128-row chunks
    const uint8_t* w2_img;   // W2^ image [0][k][p][r < rows2][32], Cout rows, K = hidden channels
    const float* b1;         // [H] fp32 or nullptr
    const float* b2;         // [Cout] fp32 or nullptr
    uint8_t* y;              // [N, Cout, G]
    int* status;
    long long N;
    int Cin, H, Cout;
    int nK1;                 // 32-channel chunks of Cin (resident x slots)
    int n_hc;                // 128-row hidden chunks
    int nK2;                 // 32-channel chunks of H (layer-2 K chunks)
    int rows2;               // rows of a W2^ sub-block (Cout rounded up to 8)
    int n_tiles;             // token tiles
    int stages;              // weight ring depth (units)
    unsigned long long timeout_ns;
    long long inject_stop;   // test hook: x chunks issued per CTA before the producer stops; -1 = never
    int w_early;             // weights may be loaded before griddepcontrol.wait (TcParams::w_early)
    int pf;                  // L2 prefetch distance of x, in tiles of this CTA (0 = off)
    int l2hint;              // L2 eviction priorities on the copies (TcParams::l2hint)
};

namespace mlp {

constexpr int kMaxK1 = 8;                              // resident x slots
constexpr int kHK = kMmaM / kChunkK;                   // K32 chunks of H^ per hidden chunk (4)
constexpr int kUnitBytes = 2 * kMmaM * kPlaneRowBytes;  // one weight unit: 2 planes x 128 rows x 64 B
constexpr int kMaxStages = 12;

template <int G>
struct Cfg {
    using S = tc::Shape<G, 2>;
    static constexpr int kUnits = G / 2;               // weight units per 32-channel chunk
    static constexpr int TGM = 32 / G;                 // tokens per TMEM load of a hidden chunk
    static constexpr int NGR = S::BN / TGM;            // such groups per token tile (8)
    // The hidden epilogue runs on 12 warps, 3 per TMEM lane quarter: the 8 epilogue warps
    // and the 4 DFT warps (which transform x once per tile and are free otherwise).  Warp
    // part j in {0, 1, 2} of a quarter takes groups j, j + 3, j + 6.
    static constexpr int kParts = 3;
    static constexpr int kHiddenThreads = 4 * kParts * 32;
    static_assert(TGM % 2 == 0 && S::BN % TGM == 0, "hidden epilogue groups");
};

// Weight unit u of a 32-channel chunk: planes 0 and 1 (the real frequencies 0 and G/2)
// for u = 0, planes 2u and 2u+1 (Re and Im of frequency u) for u >= 1.  `a_lo`: low half
// of the descriptor of the unit's first plane; `wsub16`: one plane's bytes / 16; `b_lo`:
// the spectrum chunk's slots.  Adds the unit's products for one K step into D.
template <int G, class T16>
__device__ __forceinline__ void issue_unit(int u, uint32_t d_base, uint32_t a_lo, uint32_t wsub16, uint32_t b_lo,
                                           int ks, uint32_t acc0) {
    using S = tc::Shape<G, 2>;
    constexpr uint32_t ID = idesc_f16kind_f32(kMmaM, S::BN, Io16<T16>::kUmmaFormat, false);
    constexpr uint32_t ID2 = idesc_f16kind_f32(kMmaM, G > 2 ? 2 * S::BN : S::BN, Io16<T16>::kUmmaFormat, false);
    auto A = [&](int pl) { return ptx::sdesc_sw64_from_lo(a_lo + static_cast<uint32_t>(pl) * wsub16 + ks * 2); };
    auto B = [&](int slot) { return ptx::sdesc_sw64_from_lo(b_lo + (slot * S::PLANE_BYTES + ks * 32) / 16); };
    auto D = [&](int pl) { return d_base + static_cast<uint32_t>(pl * S::BN); };
    if (u == 0) {
        ptx::umma_f16(D(0), A(0), B(0), ID, acc0);
        ptx::umma_f16(D(1), A(1), B(1), ID, acc0);
    } else {
        const int s = pair_first_slot(u);
        ptx::umma_f16(D(2 * u), A(0), B(s + 1), ID2, acc0);   // [Dr|Di] += Wr [Xr; Xi]
        ptx::umma_f16(D(2 * u), A(1), B(s), ID2, 1u);         // [Dr|Di] += Wi [-Xi; Xr]
    }
}

// Epilogue of one hidden chunk, warp (q, part): hidden rows 32q .. 32q+31 of the chunk
// (TMEM lane quarter q, one row per lane), token groups part, part + 3, ... of TGM tokens.
// Per pair of tokens (packed as fx2): irDFT of the G planes + b1, GELU, rDFT, and the G
// spectrum values written as the pair slots of H^ into K32 chunk q of `hbuf` (lane = K
// column, one 2-byte store per token and slot: a warp fills one 64-byte row).  Arrives on
// `acc1_empty` once its last TMEM load has landed.
template <int G, class T16>
__device__ __forceinline__ void hidden_chunk(const MlpParams& p, uint32_t acc1, int q, int part, int lane, int hc,
                                             uint8_t* hbuf, uint32_t acc1_empty) {
    using C = Cfg<G>;
    using S = typename C::S;
    constexpr int TGM = C::TGM;
    const int j = hc * kMmaM + q * 32 + lane;                   // hidden channel of this lane
    const bool chunk_used = hc * kHK + q < p.nK2;               // layer 2 reads this K32 chunk
    const float b = (p.b1 != nullptr && j < p.H) ? p.b1[j] : 0.0f;
    const uint32_t lane_addr = acc1 + (static_cast<uint32_t>(q * 32) << 16);
    uint8_t* hsub = hbuf + static_cast<size_t>(q) * S::SPEC_BYTES;
    const int piece = lane >> 3, in_piece = (lane & 7) * 2;
#pragma unroll 1
    for (int g = part; g < C::NGR; g += C::kParts) {
        uint32_t r[G][TGM];
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_ld_32x32b<TGM>(lane_addr + pl * S::BN + g * TGM, r[pl]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_regs_ready<TGM>(r[pl]);
        if (g + C::kParts >= C::NGR) {
            ptx::tc_fence_before();
            ptx::mbar_arrive(acc1_empty);   // acc1 no longer needed by this thread
        }
        if (!chunk_used) continue;
#pragma unroll
        for (int t = 0; t < TGM; t += 2) {
            fx2 z[G], hv[G], sp[G];
#pragma unroll
            for (int pl = 0; pl < G; ++pl) z[pl] = fx2(__uint_as_float(r[pl][t]), __uint_as_float(r[pl][t + 1]));
            z[0] += fx2(b, b);   // the DC term appears with weight 1 in every group element
            RealIdft<G, fx2>::run(z, hv);
#pragma unroll
            for (int gg = 0; gg < G; ++gg) hv[gg] = gelu2(hv[gg]);
            rdft_planes<G>(hv, sp);
            // rows tt (even) and tt + 1 share the SWIZZLE_64B piece permutation
            const int tt = g * TGM + t;
            uint8_t* row = hsub + tt * kPlaneRowBytes + ((piece ^ ((tt >> 1) & 3)) << 4) + in_piece;
            auto put = [&](int slot, uint32_t w) {
                uint8_t* d = row + slot * S::PLANE_BYTES;
                *reinterpret_cast<uint16_t*>(d) = static_cast<uint16_t>(w & 0xFFFFu);
                *reinterpret_cast<uint16_t*>(d + kPlaneRowBytes) = static_cast<uint16_t>(w >> 16);
            };
            put(0, Io16<T16>::pack(sp[0].x, sp[0].y));
            put(1, Io16<T16>::pack(sp[1].x, sp[1].y));
#pragma unroll
            for (int k = 1; k < G / 2; ++k) {
                const uint32_t re = Io16<T16>::pack(sp[2 * k].x, sp[2 * k].y);
                const uint32_t im = Io16<T16>::pack(sp[2 * k + 1].x, sp[2 * k + 1].y);
                const int s = pair_first_slot(k);
                put(s, im ^ 0x80008000u);   // exact: rounding to nearest even is symmetric
                put(s + 1, re);
                put(s + 2, im);
            }
        }
    }
}

}  // namespace mlp

template <int G, class T16>
__global__ void __launch_bounds__(tc::kThreads, 1)
    eqlin_mlp_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const MlpParams p) {
    using C = mlp::Cfg<G>;
    using S = typename C::S;
    constexpr int U = C::kUnits;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align_1k(smem_raw);

    const int NS = p.stages, nK1 = p.nK1;
    uint8_t* xslot0 = smem;                                                   // nK1 x chunks / X^
    uint8_t* hbuf = xslot0 + static_cast<size_t>(nK1) * S::SPEC_BYTES;         // H^ of one hidden chunk
    uint8_t* wring0 = hbuf + static_cast<size_t>(mlp::kHK) * S::SPEC_BYTES;    // weight units
    uint64_t* bars = reinterpret_cast<uint64_t*>(wring0 + static_cast<size_t>(NS) * mlp::kUnitBytes);
    tc::Ctl* ctl = reinterpret_cast<tc::Ctl*>(bars + 2 * mlp::kMaxK1 + 2 * NS + 9);

    auto bar_x_full = [&](int c) { return ptx::smem_u32(bars + c); };
    auto bar_xhat = [&](int c) { return ptx::smem_u32(bars + mlp::kMaxK1 + c); };
    auto bar_w_full = [&](int s) { return ptx::smem_u32(bars + 2 * mlp::kMaxK1 + s); };
    auto bar_w_empty = [&](int s) { return ptx::smem_u32(bars + 2 * mlp::kMaxK1 + NS + s); };
    uint64_t* b0 = bars + 2 * mlp::kMaxK1 + 2 * NS;
    const uint32_t bar_acc1_full = ptx::smem_u32(b0 + 0), bar_acc1_empty = ptx::smem_u32(b0 + 1);
    const uint32_t bar_h_full = ptx::smem_u32(b0 + 2), bar_h_empty = ptx::smem_u32(b0 + 3);
    const uint32_t bar_acc2_full = ptx::smem_u32(b0 + 4), bar_acc2_empty = ptx::smem_u32(b0 + 5);
    const uint32_t bar_x_free = ptx::smem_u32(b0 + 6), bar_drain = ptx::smem_u32(b0 + 7);
    const uint32_t s_xslot0 = ptx::smem_u32(xslot0), s_hbuf = ptx::smem_u32(hbuf), s_wring0 = ptx::smem_u32(wring0);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // weight units per tile, in MMA order: for each hidden chunk hc, its layer-1 units
    // (c, u), then the layer-2 units (k, u) of hc - 1; after the last chunk, its layer-2 units
    const int w1_units = nK1 * U;
    auto w2_units = [&](int hc) { return min(mlp::kHK, p.nK2 - hc * mlp::kHK) * U; };
    const int units_per_tile = p.n_hc * w1_units + p.nK2 * U;

    if (threadIdx.x == 0) {
        for (int c = 0; c < nK1; ++c) {
            ptx::mbar_init(bar_x_full(c), 1);
            ptx::mbar_init(bar_xhat(c), 128);
        }
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(bar_w_full(s), 1);
            ptx::mbar_init(bar_w_empty(s), 1);
        }
        ptx::mbar_init(bar_acc1_full, 1);
        ptx::mbar_init(bar_acc1_empty, C::kHiddenThreads);
        ptx::mbar_init(bar_h_full, C::kHiddenThreads);
        ptx::mbar_init(bar_h_empty, 1);
        ptx::mbar_init(bar_acc2_full, 1);
        ptx::mbar_init(bar_acc2_empty, tc::kEpiThreads);
        ptx::mbar_init(bar_x_free, 1);
        ptx::mbar_init(bar_drain, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == tc::kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), S::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == tc::kWarpProducer && lane == 0) ptx::prefetch_tmap(&tmap_x);
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const uint32_t acc1 = tmem_base, acc2 = tmem_base + static_cast<uint32_t>(S::ACC_COLS);
    const bool hint = p.l2hint != 0;
    const uint64_t pol_w = hint ? ptx::l2_policy_evict_last() : 0ull, pol_x = hint ? ptx::l2_policy_evict_first() : 0ull;

    // source of weight unit i (0 <= i < units_per_tile) of a tile, and its bytes
    auto unit_src = [&](int i, uint32_t* bytes) -> const uint8_t* {
        for (int hc = 0; hc <= p.n_hc; ++hc) {
            if (hc < p.n_hc) {
                if (i < w1_units) {
                    const int c = i / U, u = i % U;
                    *bytes = mlp::kUnitBytes;
                    return p.w1_img + (static_cast<size_t>(hc * nK1 + c) * G + 2 * u) * (kMmaM * kPlaneRowBytes);
                }
                i -= w1_units;
            }
            if (hc > 0) {
                const int n2 = w2_units(hc - 1);
                if (i < n2) {
                    const int k = (hc - 1) * mlp::kHK + i / U, u = i % U;
                    *bytes = 2u * static_cast<uint32_t>(p.rows2) * kPlaneRowBytes;
                    return p.w2_img + (static_cast<size_t>(k) * G + 2 * u) * (static_cast<size_t>(p.rows2) * kPlaneRowBytes);
                }
                i -= n2;
            }
        }
        *bytes = 0;
        return nullptr;
    };
    // Weights no kernel of the stream writes (p.w_early): the first ring stages are filled
    // while the previous kernel drains; the loop below skips issuing those units.
    int w_prefilled = 0;
    if (p.w_early && warp == tc::kWarpProducer && lane == 0 && blockIdx.x < p.n_tiles) {
        const int pre = min(NS, units_per_tile);
        for (int j = 0; j < pre; ++j) {
            uint32_t bytes;
            const uint8_t* src = unit_src(j, &bytes);
            ptx::mbar_arrive_expect_tx(bar_w_full(j), bytes);
            ptx::bulk_load_h(s_wring0 + j * mlp::kUnitBytes, src, bytes, bar_w_full(j), hint, pol_w);
        }
        w_prefilled = pre;
    }
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();

    if (warp == tc::kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int tiles_loaded = 0, last_tile_chunks = 0;
            long long issued_x = 0, issued_w = 0;
            int ws = 0;
            uint32_t wph = 0;
            bool ok = true;
            auto prefetch_tile = [&](long long t) {
                if (t >= p.n_tiles) return;
                const int n0 = static_cast<int>(t) * S::BN;
                for (int c = 0; c < nK1; ++c)
#pragma unroll
                    for (int bx = 0; bx < S::NBOX; ++bx)
                        ptx::tma_prefetch_l2_2d(&tmap_x, c * S::XROW_ELEMS + bx * S::BOX_ELEMS, n0);
            };
            for (int j = 1; j < p.pf; ++j) prefetch_tile(blockIdx.x + static_cast<long long>(j) * gridDim.x);
            int ti = 0;
            for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++ti) {
                if (p.pf > 0) prefetch_tile(tile + static_cast<long long>(p.pf) * gridDim.x);
                if (!tc::wait_bounded(bar_x_free, (static_cast<uint32_t>(ti) & 1u) ^ 1u, ctl, p.status,
                                      p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const int n0 = tile * S::BN;
                last_tile_chunks = 0;
                for (int c = 0; c < nK1; ++c) {
                    if (issued_x == p.inject_stop) {   // test hook (failure detection)
                        ok = false;
                        break;
                    }
                    const uint32_t dst = s_xslot0 + c * S::SPEC_BYTES;
                    ptx::mbar_arrive_expect_tx(bar_x_full(c), S::XCHUNK_BYTES);
#pragma unroll
                    for (int bx = 0; bx < S::NBOX; ++bx)
                        ptx::tma_load_2d_h(dst + bx * (S::BN * S::BOX_ELEMS * 2), &tmap_x,
                                           c * S::XROW_ELEMS + bx * S::BOX_ELEMS, n0, bar_x_full(c), hint, pol_x);
                    ++issued_x;
                    ++last_tile_chunks;
                }
                if (!ok) break;
                ++tiles_loaded;
                for (int i = 0; i < units_per_tile; ++i) {
                    if (issued_w < w_prefilled) {   // issued before griddepcontrol.wait
                        ++issued_w;
                        if (++ws == NS) { ws = 0; wph ^= 1u; }
                        continue;
                    }
                    if (!tc::wait_bounded(bar_w_empty(ws), wph ^ 1u, ctl, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    uint32_t bytes;
                    const uint8_t* src = unit_src(i, &bytes);
                    ptx::mbar_arrive_expect_tx(bar_w_full(ws), bytes);
                    ptx::bulk_load_h(s_wring0 + ws * mlp::kUnitBytes, src, bytes, bar_w_full(ws), hint, pol_w);
                    ++issued_w;
                    if (++ws == NS) { ws = 0; wph ^= 1u; }
                }
            }
            // drain (bounded, blind to the abort flag): every copy issued lands before exit
            for (int c = 0; c < nK1; ++c) {
                const int uses = tiles_loaded + (c < last_tile_chunks && last_tile_chunks < nK1 ? 1 : 0);
                if (uses > 0) tc::drain_wait(bar_x_full(c), static_cast<uint32_t>((uses - 1) & 1), p.status, p.timeout_ns);
            }
            const long long w_total = issued_w > w_prefilled ? issued_w : w_prefilled;
            for (int s = 0; s < NS; ++s) {
                const long long times = w_total > s ? (w_total - s + NS - 1) / NS : 0;
                if (times > 0)
                    tc::drain_wait(bar_w_full(s), static_cast<uint32_t>((times - 1) & 1), p.status, p.timeout_ns);
            }
        }
    } else if (warp == tc::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t wsub1_16 = (kMmaM * kPlaneRowBytes) >> 4;
            const uint32_t wsub2_16 = (static_cast<uint32_t>(p.rows2) * kPlaneRowBytes) >> 4;
            bool ok = true;
            int ws = 0;
            uint32_t wph = 0;
            long long uc = 0;   // hidden chunks issued (all tiles)
            // layer-2 products of hidden chunk hc (global count u) into acc2
            auto layer2 = [&](int hc, long long u, int ti) -> bool {
                if (!tc::wait_bounded(bar_h_full, static_cast<uint32_t>(u & 1), ctl, p.status, p.timeout_ns)) return false;
                if (hc == 0 &&
                    !tc::wait_bounded(bar_acc2_empty, (static_cast<uint32_t>(ti) & 1u) ^ 1u, ctl, p.status, p.timeout_ns))
                    return false;
                ptx::tc_fence_after();
                const int nk = min(mlp::kHK, p.nK2 - hc * mlp::kHK);
                for (int kk = 0; kk < nk; ++kk) {
                    const uint32_t b_lo = ptx::sdesc_sw64_lo(s_hbuf + kk * S::SPEC_BYTES);
                    for (int u2 = 0; u2 < U; ++u2) {
                        if (!tc::wait_bounded(bar_w_full(ws), wph, ctl, p.status, p.timeout_ns)) return false;
                        ptx::tc_fence_after();
                        const uint32_t a_lo = ptx::sdesc_sw64_lo(s_wring0 + ws * mlp::kUnitBytes);
#pragma unroll
                        for (int ks = 0; ks < kChunkK / 16; ++ks)
                            mlp::issue_unit<G, T16>(u2, acc2, a_lo, wsub2_16, b_lo, ks,
                                                    (hc > 0 || kk > 0 || ks > 0) ? 1u : 0u);
                        ptx::umma_commit(bar_w_empty(ws));
                        if (++ws == NS) { ws = 0; wph ^= 1u; }
                    }
                }
                ptx::umma_commit(bar_h_empty);   // H^ reusable once these products finish
                return true;
            };
            int ti = 0;
            for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++ti) {
                for (int hc = 0; ok && hc < p.n_hc; ++hc, ++uc) {
                    // layer 1 of hc into acc1 (free once the epilogue has loaded hc - 1)
                    if (!tc::wait_bounded(bar_acc1_empty, static_cast<uint32_t>(uc & 1) ^ 1u, ctl, p.status,
                                          p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    for (int c = 0; ok && c < nK1; ++c) {
                        if (hc == 0 &&
                            !tc::wait_bounded(bar_xhat(c), static_cast<uint32_t>(ti) & 1u, ctl, p.status, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        const uint32_t b_lo = ptx::sdesc_sw64_lo(s_xslot0 + c * S::SPEC_BYTES);
                        for (int u1 = 0; u1 < U; ++u1) {
                            if (!tc::wait_bounded(bar_w_full(ws), wph, ctl, p.status, p.timeout_ns)) {
                                ok = false;
                                break;
                            }
                            ptx::tc_fence_after();
                            const uint32_t a_lo = ptx::sdesc_sw64_lo(s_wring0 + ws * mlp::kUnitBytes);
#pragma unroll
                            for (int ks = 0; ks < kChunkK / 16; ++ks)
                                mlp::issue_unit<G, T16>(u1, acc1, a_lo, wsub1_16, b_lo, ks, (c > 0 || ks > 0) ? 1u : 0u);
                            ptx::umma_commit(bar_w_empty(ws));
                            if (++ws == NS) { ws = 0; wph ^= 1u; }
                        }
                    }
                    if (!ok) break;
                    ptx::umma_commit(bar_acc1_full);
                    if (hc == p.n_hc - 1) ptx::umma_commit(bar_x_free);   // x slots reusable
                    // layer 2 of the previous hidden chunk (its H^ is written by now or soon)
                    if (hc > 0 && !layer2(hc - 1, uc - 1, ti)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                if (!layer2(p.n_hc - 1, uc - 1, ti)) {
                    ok = false;
                    break;
                }
                ptx::umma_commit(bar_acc2_full);
            }
            ptx::umma_commit(bar_drain);
            tc::drain_wait(bar_drain, 0, p.status, p.timeout_ns);
        }
    } else if (warp >= tc::kWarpDft0) {
        // ------------------------------------------------------------ DFT warps
        // per tile: the x chunks' DFT, then their part of each hidden chunk's epilogue
        const int dft_tid = threadIdx.x - tc::kWarpDft0 * 32;
        long long uc = 0;
        bool ok = true;
        int ti = 0;
        for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++ti) {
            for (int c = 0; c < nK1; ++c) {
                const bool got = tc::wait_bounded(bar_x_full(c), static_cast<uint32_t>(ti) & 1u, ctl, p.status,
                                                  p.timeout_ns);
                if (!ptx::named_bar_and(tc::kBarDft, 128, got)) {
                    ok = false;
                    break;
                }
                tc::dft_chunk<G, 2, T16>(xslot0 + static_cast<size_t>(c) * S::SPEC_BYTES, dft_tid);
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(bar_xhat(c));
            }
            for (int hc = 0; ok && hc < p.n_hc; ++hc, ++uc) {
                bool got = tc::wait_bounded(bar_acc1_full, static_cast<uint32_t>(uc & 1), ctl, p.status, p.timeout_ns);
                got = got && tc::wait_bounded(bar_h_empty, static_cast<uint32_t>(uc & 1) ^ 1u, ctl, p.status,
                                              p.timeout_ns);
                if (!ptx::named_bar_and(tc::kBarDft, 128, got)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                mlp::hidden_chunk<G, T16>(p, acc1, warp & 3, 2, lane, hc, hbuf, bar_acc1_empty);
                ptx::fence_proxy_async_smem();   // H^ visible to the tensor cores
                ptx::mbar_arrive(bar_h_full);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const int q = warp & 3, half = warp >> 2;
        TcParams out{};   // the output epilogue is the single layer's, with direct stores
        out.y = p.y;
        out.bias = p.b2;
        out.N = p.N;
        out.Cout = p.Cout;
        out.ybufs = 0;
        out.act = kActNone;
        int ybuf = 0;
        long long uc = 0;
        bool ok = true;
        int ti = 0;
        for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x, ++ti) {
            for (int hc = 0; hc < p.n_hc; ++hc, ++uc) {
                bool got = tc::wait_bounded(bar_acc1_full, static_cast<uint32_t>(uc & 1), ctl, p.status, p.timeout_ns);
                got = got && tc::wait_bounded(bar_h_empty, static_cast<uint32_t>(uc & 1) ^ 1u, ctl, p.status,
                                              p.timeout_ns);
                if (!ptx::named_bar_and(tc::kBarEpi, tc::kEpiThreads, got)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                mlp::hidden_chunk<G, T16>(p, acc1, q, half, lane, hc, hbuf, bar_acc1_empty);   // parts 0, 1
                ptx::fence_proxy_async_smem();   // H^ visible to the tensor cores
                ptx::mbar_arrive(bar_h_full);
            }
            if (!ok) break;
            const bool got = tc::wait_bounded(bar_acc2_full, static_cast<uint32_t>(ti) & 1u, ctl, p.status,
                                              p.timeout_ns);
            if (!ptx::named_bar_and(tc::kBarEpi, tc::kEpiThreads, got)) break;
            ptx::tc_fence_after();
            if (q * 32 < p.Cout)
                tc::epilogue_tile<G, 2, T16>(out, nullptr, acc2, q, half, lane, static_cast<long long>(tile) * S::BN, 0,
                                             nullptr, ybuf);
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_acc2_empty);
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == tc::kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ fp32 path
// The block for fp32 I/O on CUDA cores, in float64 throughout (as eqlin_fwd_f32_kernel):
// block = 8 warps over 8 tokens; the spectra of the tokens' inputs and of their hidden
// activation stay in shared memory ([8][G][Cin] and [8][G][H] doubles), and y is rounded
// once.  Warp = token; lanes stride over the hidden channels, then over the outputs.
// w1_f64 [G][Cin][H] and w2_f64 [G][H][Cout] are the scaled planes of eqlin_layout.h.
template <int G>
__global__ void __launch_bounds__(kF32Threads, 1)
    eqlin_mlp_f32_kernel(const float* __restrict__ x, const double* __restrict__ w1_f64,
                         const double* __restrict__ b1_f64, const double* __restrict__ w2_f64,
                         const double* __restrict__ b2_f64, float* __restrict__ y, long long N, int Cin, int H,
                         int Cout) {
    extern __shared__ double sm[];
    double* xs = sm;                                   // [kF32Tokens][G][Cin]
    double* hs = sm + static_cast<size_t>(kF32Tokens) * G * Cin;   // [kF32Tokens][G][H]
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
    const int t = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long n = n0 + t;
    // one per-frequency contraction, irDFT and bias: the single layer's arithmetic
    auto layer = [&](const double* in, int K, const double* w, const double* bias, int O, int o, double (&out)[G]) {
        double z[G];
#pragma unroll
        for (int p = 0; p < G; ++p) z[p] = 0.0;
        for (int i = 0; i < K; ++i) {
            double xv[G], wv[G];
#pragma unroll
            for (int p = 0; p < G; ++p) {
                xv[p] = in[p * K + i];
                wv[p] = w[(static_cast<size_t>(p) * K + i) * O + o];
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
        z[0] += bias != nullptr ? bias[o] : 0.0;
        RealIdft<G, double>::run(z, out);
    };
    const double* xt = xs + static_cast<size_t>(t) * G * Cin;
    double* ht = hs + static_cast<size_t>(t) * G * H;
    for (int j = lane; j < H; j += 32) {
        double hv[G], pl[G];
        layer(xt, Cin, w1_f64, b1_f64, H, j, hv);
#pragma unroll
        for (int g = 0; g < G; ++g) hv[g] = gelu(hv[g]);
        rdft_planes<G, double>(hv, pl);
#pragma unroll
        for (int p = 0; p < G; ++p) ht[p * H + j] = pl[p];
    }
    __syncwarp();   // a warp reads only its own token's hidden spectrum
    if (n >= N) return;
    for (int o = lane; o < Cout; o += 32) {
        double yv[G];
        layer(ht, H, w2_f64, b2_f64, Cout, o, yv);
        float* dst = y + (n * Cout + o) * G;
#pragma unroll
        for (int g = 0; g < G; ++g) dst[g] = static_cast<float>(yv[g]);
    }
}

}  // namespace eqlin
