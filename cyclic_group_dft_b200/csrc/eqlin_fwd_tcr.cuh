// eqlin_fwd_tcr.cuh -- tokens-on-N fused forward with the input spectrum resident
// across output chunks (layers with Cout > 128).
//
// Same operation and arithmetic as eqlin_fwd_tc.cuh (page "Flash EQ-Linear:
// Accelerating Equivariant Linear Layers via Group-wise Discrete Fourier Transform",
// sections "Enfoque Algoritmico" and "Implementacion").  There a work item is one
// (token tile, 128-row output chunk) pair, so a layer with n_oc output chunks loads and
// transforms every x chunk n_oc times.  Here a work item is a whole token tile: its nK
// x chunks are loaded and transformed once into nK resident smem slots, then the MMAs
// of all n_oc output chunks read them while the weight chunks (oc, c) stream through a
// ring.  The two TMEM accumulators alternate between output chunks, so the MMAs of
// chunk oc+1 overlap the epilogue of chunk oc.  The next tile's x chunks are loaded once
// the last MMA of the tile has completed.
//
// Roles (warps as in eqlin_fwd_tc.cuh):
//   warp 12     producer: x chunks of a tile into their slots (TMA), weight chunks into
//               the ring (bulk copies)
//   warps 8-11  DFT of each slot in place (tc::dft_chunk)
//   warp 13     MMA issuer + TMEM owner
//   warps 0-7   epilogue (tc::epilogue_tile), per (tile, output chunk)
// Waits are bounded as in eqlin_fwd_tc.cuh.
#pragma once

#include <cstdint>

#include "eqlin_fwd_tc.cuh"
#include "eqlin_layout.h"
#include "io16.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

namespace tcr {
constexpr int kMaxK = 8;   // resident x slots (32-channel chunks)
}

// p.n_work = token tiles, p.stages = weight ring depth.
template <int G, class T16>
__global__ void __launch_bounds__(tc::kThreads, 1)
    eqlin_fwd_tcr_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_y,
                         const TcParams p) {
    using S = tc::Shape<G, 2>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align_1k(smem_raw);

    const int NS = p.stages, nK = p.nK;
    uint8_t* ystage0 = smem;                                          // y staging per epilogue warp
    uint8_t* xslot0 = ystage0 + tc::kEpiWarps * static_cast<size_t>(p.ystage_bytes);
    uint8_t* wring0 = xslot0 + static_cast<size_t>(nK) * S::SPEC_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(wring0 + static_cast<size_t>(NS) * S::WSTAGE_BYTES);
    tc::Ctl* ctl = reinterpret_cast<tc::Ctl*>(bars + 2 * tcr::kMaxK + 2 * NS + 6);

    auto bar_x_full = [&](int c) { return ptx::smem_u32(bars + c); };
    auto bar_xhat = [&](int c) { return ptx::smem_u32(bars + tcr::kMaxK + c); };
    auto bar_w_full = [&](int s) { return ptx::smem_u32(bars + 2 * tcr::kMaxK + s); };
    auto bar_w_empty = [&](int s) { return ptx::smem_u32(bars + 2 * tcr::kMaxK + NS + s); };
    auto bar_acc_full = [&](int a) { return ptx::smem_u32(bars + 2 * tcr::kMaxK + 2 * NS + a); };
    auto bar_acc_empty = [&](int a) { return ptx::smem_u32(bars + 2 * tcr::kMaxK + 2 * NS + 2 + a); };
    const uint32_t bar_x_free = ptx::smem_u32(bars + 2 * tcr::kMaxK + 2 * NS + 4);
    const uint32_t bar_drain = ptx::smem_u32(bars + 2 * tcr::kMaxK + 2 * NS + 5);
    const uint32_t s_xslot0 = ptx::smem_u32(xslot0), s_wring0 = ptx::smem_u32(wring0);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int c = 0; c < nK; ++c) {
            ptx::mbar_init(bar_x_full(c), 1);
            ptx::mbar_init(bar_xhat(c), 128);
        }
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(bar_w_full(s), 1);
            ptx::mbar_init(bar_w_empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(bar_acc_full(a), 1);
            ptx::mbar_init(bar_acc_empty(a), tc::kEpiThreads);
        }
        ptx::mbar_init(bar_x_free, 1);
        ptx::mbar_init(bar_drain, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == tc::kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), S::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (warp == tc::kWarpProducer && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_y);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const bool hint = p.l2hint != 0;
    const uint64_t pol_w = hint ? ptx::l2_policy_evict_last() : 0ull, pol_x = hint ? ptx::l2_policy_evict_first() : 0ull;
    // Weights that no kernel of the stream writes (p.w_early): the first ring stages are
    // filled with the first tile's weight chunks while the previous kernel drains.  The
    // ring order is the same as below, which then skips issuing those chunks.
    int w_prefilled = 0;
    if (p.w_early && warp == tc::kWarpProducer && lane == 0 && blockIdx.x < p.n_work) {
        const int pre = min(NS, p.n_oc * nK);
        for (int j = 0; j < pre; ++j) {
            ptx::mbar_arrive_expect_tx(bar_w_full(j), S::WSTAGE_BYTES);
            ptx::bulk_load_h(s_wring0 + j * S::WSTAGE_BYTES, p.w_img + static_cast<size_t>(j) * S::WSTAGE_BYTES,
                             S::WSTAGE_BYTES, bar_w_full(j), hint, pol_w);
        }
        w_prefilled = pre;
    }
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();

    if (warp == tc::kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int tiles_loaded = 0;          // tiles whose x chunks were all issued
            int last_tile_chunks = 0;      // x chunks issued for the last (possibly partial) tile
            long long issued_x = 0, issued_w = 0;
            int ws = 0;
            uint32_t wph = 0;
            bool ok = true;
            int ti = 0;
            // x chunks of token tile t into L2 (a hint: the loads below still bring them)
            auto prefetch_tile = [&](long long t) {
                if (t >= p.n_work) return;
                const int n0 = static_cast<int>(t) * S::BN;
                for (int c = 0; c < nK; ++c)
#pragma unroll
                    for (int bx = 0; bx < S::NBOX; ++bx)
                        ptx::tma_prefetch_l2_2d(&tmap_x, c * S::XROW_ELEMS + bx * S::BOX_ELEMS, n0);
            };
            for (int j = 1; j < p.pf; ++j) prefetch_tile(blockIdx.x + static_cast<long long>(j) * gridDim.x);
            for (int tile = blockIdx.x; ok && tile < p.n_work; tile += gridDim.x, ++ti) {
                if (p.pf > 0) prefetch_tile(tile + static_cast<long long>(p.pf) * gridDim.x);
                // the slots are free once every MMA of the previous tile has completed
                if (!tc::wait_bounded(bar_x_free, (static_cast<uint32_t>(ti) & 1u) ^ 1u, ctl, p.status,
                                      p.timeout_ns)) {
                    ok = false;
                    break;
                }
                const int n0 = tile * S::BN;
                last_tile_chunks = 0;
                for (int c = 0; c < nK; ++c) {
                    // test hook (failure detection): stop issuing after inject_stop x chunks
                    if (issued_x == p.inject_stop) {
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
                for (int oc = 0; ok && oc < p.n_oc; ++oc) {
                    for (int c = 0; c < nK; ++c) {
                        if (issued_w < w_prefilled) {   // issued before griddepcontrol.wait
                            ++issued_w;
                            if (++ws == NS) { ws = 0; wph ^= 1u; }
                            continue;
                        }
                        if (!tc::wait_bounded(bar_w_empty(ws), wph ^ 1u, ctl, p.status, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        ptx::mbar_arrive_expect_tx(bar_w_full(ws), S::WSTAGE_BYTES);
                        ptx::bulk_load_h(s_wring0 + ws * S::WSTAGE_BYTES,
                                       p.w_img + static_cast<size_t>(oc * nK + c) * S::WSTAGE_BYTES,
                                       S::WSTAGE_BYTES, bar_w_full(ws), hint, pol_w);
                        ++issued_w;
                        if (++ws == NS) { ws = 0; wph ^= 1u; }
                    }
                }
            }
            // drain (bounded, blind to the abort flag): every copy issued lands before exit.
            // x slot c completed (tiles_loaded) phases, plus one more if the last, partial
            // tile issued it.
            for (int c = 0; c < nK; ++c) {
                const int uses = tiles_loaded + (c < last_tile_chunks && last_tile_chunks < nK ? 1 : 0);
                if (uses > 0) tc::drain_wait(bar_x_full(c), static_cast<uint32_t>((uses - 1) & 1), p.status, p.timeout_ns);
            }
            // chunks prefilled before the wait are in flight even if the loop stopped early
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
            constexpr uint32_t ID = idesc_f16kind_f32(kMmaM, S::BN, Io16<T16>::kUmmaFormat, false);
            constexpr uint32_t ID2 = idesc_f16kind_f32(kMmaM, G > 2 ? 2 * S::BN : S::BN, Io16<T16>::kUmmaFormat, false);
            constexpr uint32_t wsub16 = (kMmaM * kPlaneRowBytes) >> 4;
            bool ok = true;
            int it = 0, ws = 0, ti = 0;
            uint32_t wph = 0;
            for (int tile = blockIdx.x; ok && tile < p.n_work; tile += gridDim.x, ++ti) {
                for (int oc = 0; ok && oc < p.n_oc; ++oc, ++it) {
                    const int abuf = it & 1;
                    if (!tc::wait_bounded(bar_acc_empty(abuf), (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u, ctl,
                                          p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t acc_base = tmem_base + static_cast<uint32_t>(abuf * S::ACC_COLS);
                    for (int c = 0; c < nK; ++c) {
                        if (oc == 0 &&
                            !tc::wait_bounded(bar_xhat(c), static_cast<uint32_t>(ti) & 1u, ctl, p.status, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        if (!tc::wait_bounded(bar_w_full(ws), wph, ctl, p.status, p.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        ptx::tc_fence_after();
                        const uint32_t a_lo = ptx::sdesc_sw64_lo(s_wring0 + ws * S::WSTAGE_BYTES);
                        const uint32_t b_lo = ptx::sdesc_sw64_lo(s_xslot0 + c * S::SPEC_BYTES);
                        const uint32_t acc_first = c > 0 ? 1u : 0u;
#pragma unroll
                        for (int ks = 0; ks < kChunkK / 16; ++ks) {
                            const uint32_t acc0 = ks > 0 ? 1u : acc_first;
                            auto A = [&](int pl) {
                                return ptx::sdesc_sw64_from_lo(a_lo + static_cast<uint32_t>(pl) * wsub16 + ks * 2);
                            };
                            auto B = [&](int slot) {
                                return ptx::sdesc_sw64_from_lo(b_lo + (slot * S::PLANE_BYTES + ks * 32) / 16);
                            };
                            auto D = [&](int pl) { return acc_base + static_cast<uint32_t>(pl * S::BN); };
                            ptx::umma_f16(D(0), A(0), B(0), ID, acc0);
                            ptx::umma_f16(D(1), A(1), B(1), ID, acc0);
#pragma unroll
                            for (int k = 1; k < G / 2; ++k) {
                                const int pr = 2 * k, pi = 2 * k + 1, s = pair_first_slot(k);
                                ptx::umma_f16(D(pr), A(pr), B(s + 1), ID2, acc0);   // [Dr|Di] += Wr [Xr; Xi]
                                ptx::umma_f16(D(pr), A(pi), B(s), ID2, 1u);         // [Dr|Di] += Wi [-Xi; Xr]
                            }
                        }
                        ptx::umma_commit(bar_w_empty(ws));
                        if (++ws == NS) { ws = 0; wph ^= 1u; }
                    }
                    if (!ok) break;
                    ptx::umma_commit(bar_acc_full(abuf));
                }
                if (!ok) break;
                ptx::umma_commit(bar_x_free);   // the slots are reusable once these MMAs finish
            }
            ptx::umma_commit(bar_drain);
            tc::drain_wait(bar_drain, 0, p.status, p.timeout_ns);
        }
    } else if (warp >= tc::kWarpDft0) {
        // ------------------------------------------------------------ DFT warps
        const int dft_tid = threadIdx.x - tc::kWarpDft0 * 32;
        int ti = 0;
        for (int tile = blockIdx.x; tile < p.n_work; tile += gridDim.x, ++ti) {
            bool ok = true;
            for (int c = 0; c < nK; ++c) {
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
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const int half = warp >> 2;
        uint8_t* wstage = ystage0 + static_cast<size_t>(warp) * p.ystage_bytes;
        int ybuf = 0;
        int it = 0;
        bool ok = true;
        for (int tile = blockIdx.x; ok && tile < p.n_work; tile += gridDim.x) {
            for (int oc = 0; oc < p.n_oc; ++oc, ++it) {
                const int abuf = it & 1;
                const bool got = tc::wait_bounded(bar_acc_full(abuf), static_cast<uint32_t>(it >> 1) & 1u, ctl,
                                                  p.status, p.timeout_ns);
                if (!ptx::named_bar_and(tc::kBarEpi, tc::kEpiThreads, got)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                if (oc * kMmaM + (warp & 3) * 32 < p.Cout) {
                    tc::epilogue_tile<G, 2, T16>(p, &tmap_y, tmem_base + static_cast<uint32_t>(abuf * S::ACC_COLS),
                                                 warp & 3, half, lane, static_cast<long long>(tile) * S::BN, oc, wstage,
                                                 ybuf);
                }
                ptx::tc_fence_before();
                ptx::mbar_arrive(bar_acc_empty(abuf));
            }
        }
        if (lane == 0) ptx::bulk_wait_group<0>();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == tc::kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, S::TMEM_COLS);
    }
}

}  // namespace eqlin
