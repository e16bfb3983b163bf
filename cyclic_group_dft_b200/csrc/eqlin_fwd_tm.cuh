// eqlin_fwd_tm.cuh -- fused EQ-Linear forward with tokens on the MMA M dimension.
//
// Same operation and steps as eqlin_fwd_tc.cuh (page "Flash EQ-Linear: Accelerating
// Equivariant Linear Layers via Group-wise Discrete Fourier Transform", sections
// "Enfoque Algoritmico" and "Implementacion"), with the operand roles of the
// per-frequency products swapped:
//   A = X^ plane [128 tokens x 16 channels]  (M = 128 tokens)
//   B = W^ plane [NO output channels x 16]   (N = NO <= 512/G, a multiple of 32)
//   D = TMEM, lane = token, column = output channel, one plane per frequency component
// A work item (128 tokens, NO output channels) needs G MMAs per 16 input channels,
// independent of how many output channels it covers, so small Cout configurations
// issue 4-8x fewer MMAs than with tokens on N.  G*NO <= 512 TMEM columns leaves room for
// one accumulator: the MMAs of a tile wait for the epilogue of the previous tile to
// release it (the epilogue releases it as soon as its last TMEM load has landed).
//
// Roles per CTA (one per SM, persistent):
//   producer warp    TMA loads of x chunks [128 tokens x 16 channels x G] (+ the weight
//                    chunk when the weights are streamed) into a smem ring
//   DW DFT warps     in-place real DFT over G: x chunk -> G planes, K-major SWIZZLE_32B,
//                    laid out so that each 8-row group of the spectrum replaces the same
//                    rows of the input (tm::SpecLayout): a warp transforms whole groups
//                    and orders only its own reads before its writes
//   MMA warp         one thread issues tcgen05.mma: 2 real products, and per complex
//                    frequency Xr [Wr | Wi] over the Re and Im planes of D at once
//                    (N = 2*NO), then for G <= 8 Xi (-Wi) into Re (the negate-B bit) and
//                    Xi Wr into Im (N = NO), for G = 16 Xi [-Wi | Wr] from the weight
//                    image's pair slots (eqlin_layout.h, tm_weight_slots)
//   8 epilogue warps lane = token; per group of 32/G output channels: tcgen05.ld of the
//                    G planes, inverse real DFT + bias, bf16, into the warp's own
//                    SWIZZLE_64B staging tile [32 tokens x 32 columns], TMA store by the
//                    warp (rows past N and columns past Cout*G clipped); warps w and w+4
//                    split the output channels
// Waits are bounded as in eqlin_fwd_tc.cuh.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "eqlin_fwd_tc.cuh"
#include "eqlin_layout.h"
#include "group_dft.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

struct TmParams {
    const uint8_t* w_img;   // weight image, image_offset_k16 layout with NO rows per sub-block
    const float* bias;      // [Cout] fp32, or nullptr
    int* status;
    long long N;
    int Cout;
    int nK;                 // 16-channel chunks along Cin
    int NO;                 // output channels per work item (MMA N)
    int n_oc;               // output chunks
    int n_work;             // token tiles * n_oc
    int stages;
    uint32_t w_region_bytes;  // resident weights (0 when streamed)
    uint32_t w_img_bytes;
    unsigned long long timeout_ns;
    long long inject_stop;  // test hook: chunks issued per CTA before the producer stops; -1 = never
    int act;                // epilogue activation after the bias: kActNone or kActGelu
    int w_early;            // weights may be loaded before griddepcontrol.wait (TcParams::w_early)
    int pf;                 // L2 prefetch distance in work items (TcParams::pf), 0 = off
    int l2hint;             // L2 eviction priorities on the copies (TcParams::l2hint)
};

namespace tm {

constexpr int kM = 128;                          // tokens per tile (MMA M)
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kBarDft = 1;
constexpr int kBarEpi = 2;
constexpr int kYCols = 32;                       // staged y columns per group (64 B rows)
constexpr int kYRows = 32;                       // staged tokens per epilogue warp (TMA box rows)
constexpr int kYWarpBufBytes = kYRows * kYCols * 2;   // 2 KB, 512-byte aligned
constexpr int kYWarpBufs = 2;                    // per epilogue warp
constexpr int kYStageBytes = kEpiWarps * kYWarpBufs * kYWarpBufBytes;   // 32 KB

template <int G>
struct Cfg {
    // DFT warps: at most 6 keep the CTA at 16 warps (128 registers per thread; 18 warps
    // would cap it at 96).  B200: p8 C64 20.8 us with 6, 21.2 us with 4; C16 C32 123.2 us
    // with 4, 129.8 us with 6 (its DFT warps then share two SM partitions with epilogue
    // warps, whose G = 16 inverse transforms are as long as the DFT's)
    static constexpr int DW = G == 16 ? 4 : 6;
    static constexpr int kDftThreads = DW * 32;
    static constexpr int kWarpDft0 = kEpiWarps;
    static constexpr int kWarpProducer = kEpiWarps + DW;
    static constexpr int kWarpMma = kEpiWarps + DW + 1;
    static constexpr int kThreads = (kEpiWarps + DW + 2) * 32;
    static constexpr int PLANE_BYTES = kM * kRowBytes32;      // 4 KB
    static constexpr int XCHUNK_BYTES = G * PLANE_BYTES;      // 128 tokens x 16 ch x G x 2
    static constexpr int XROW_ELEMS = kChunkK16 * G;          // <= 256 elements per token row
    // G >= 8: the chunk lands as XROW_ELEMS/64 boxes of [128 rows x 128 B], SWIZZLE_128B,
    // so the DFT's reads of 4G-byte units (lanes over 4 rows x 8 channel pairs) spread
    // over all banks; G <= 4: one unswizzled box (its 16-byte units are conflict-free)
    static constexpr bool X_SW128 = G >= 8;
    static constexpr int X_BOX = X_SW128 ? 64 : XROW_ELEMS;
    static constexpr int X_NBOX = XROW_ELEMS / X_BOX;
    static constexpr int X_BOX_BYTES = kM * X_BOX * 2;
    static constexpr int NMAX = (512 / G) < 256 ? (512 / G) : 256;
    static constexpr int OG = 32 / G;                         // output channels per group
    static_assert(XROW_ELEMS <= 256, "x box");
    static_assert(XCHUNK_BYTES % 1024 == 0, "stage alignment");
};

// Spectrum layout of a chunk (the MMA's A operand, K-major SWIZZLE_32B): plane p's
// 8-row atoms (8 tokens x 16 channels, 256 B) sit SBO bytes apart, inside x box p / PPB
// at byte (p % PPB) * 256 of each 8-row block of that box.  The x chunk lands as boxes of
// [128 rows x BOX_ROW bytes], so rows 8g..8g+7 of every plane occupy exactly the bytes of
// input rows 8g..8g+7: the transform of an 8-row group writes over its own input only.
template <int G>
struct SpecLayout {
    static constexpr int BOX_ROW = Cfg<G>::X_BOX * 2;          // bytes of one x box row
    static constexpr int PPB = BOX_ROW / kRowBytes32;          // planes per box
    static constexpr int SBO = 8 * BOX_ROW;                    // bytes between 8-row atoms
    static_assert(PPB * 256 == SBO && SBO % 16 == 0, "spectrum atoms tile the x boxes");
    static constexpr uint32_t plane_offset(int p) {
        return static_cast<uint32_t>((p / PPB) * Cfg<G>::X_BOX_BYTES + (p % PPB) * 256);
    }
};

// The A-operand descriptor's constant half for SpecLayout<G> (SBO, version, SWIZZLE_32B).
template <int G>
constexpr uint32_t spec_desc_hi() {
    return (static_cast<uint32_t>(SpecLayout<G>::SBO) >> 4) | (1u << 14) | (6u << 29);
}

// --------------------------------------------------------------- DFT role
// Unit = one token row x two adjacent channels (2*G 16-bit values).  Warp w transforms the
// 8-row groups w, w + DW, ...; a group's 64 units are one warp's (two per lane), so a
// __syncwarp between its reads and its in-place writes is the only ordering the
// transform needs.  Lane mapping, chosen so that the 8 lanes of each 16-byte load pass
// hit 8 different bank groups: with SWIZZLE_128B boxes (G >= 8) lane l takes row
// 8g + l%8 and channel pairs l/8 and 4 + l/8 (one pair, eight rows per pass: eight
// different swizzle slots); with unswizzled boxes it takes pair l%8 of rows 8g + l/8 and
// 8g + 4 + l/8 (one row's contiguous units per pass).  The 32-bit spectrum stores are
// conflict-free either way.
template <int G>
__device__ __forceinline__ int dft_row(int g, int s, int lane) {
    return Cfg<G>::X_SW128 ? 8 * g + (lane & 7) : 8 * g + 4 * s + (lane >> 3);
}
template <int G>
__device__ __forceinline__ int dft_pair(int s, int lane) {
    return Cfg<G>::X_SW128 ? (lane >> 3) + 4 * s : (lane & 7);
}

template <int G, class T16>
__device__ __forceinline__ void dft_chunk(uint8_t* xs, int dft_tid) {
    using C = Cfg<G>;
    using L = SpecLayout<G>;
    constexpr int WORDS = G;
    constexpr int GROUPS = kM / 8;
    const int warp = dft_tid >> 5, lane = dft_tid & 31;
#pragma unroll 1
    for (int g = warp; g < GROUPS; g += C::DW) {
        uint32_t w[2][WORDS];
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int r = dft_row<G>(g, s, lane);
            const int pair = dft_pair<G>(s, lane);
            if constexpr (C::X_SW128) {
                // 16-byte piece c of the unit: logical byte offset pair*4G + 16c in the row,
                // box off/128, piece (off/16)%8 stored at piece ^ (row % 8)
#pragma unroll
                for (int c = 0; c < WORDS / 4; ++c) {
                    const int off = pair * (4 * G) + 16 * c;
                    const uint8_t* q =
                        xs + (off >> 7) * C::X_BOX_BYTES + r * 128 + ((((off >> 4) & 7) ^ (r & 7)) << 4);
                    const uint4 v = *reinterpret_cast<const uint4*>(q);
                    w[s][4 * c + 0] = v.x;
                    w[s][4 * c + 1] = v.y;
                    w[s][4 * c + 2] = v.z;
                    w[s][4 * c + 3] = v.w;
                }
            } else {
                const uint8_t* src = xs + r * L::BOX_ROW + pair * (4 * G);
                if constexpr (WORDS == 2) {
                    const uint2 v = *reinterpret_cast<const uint2*>(src);
                    w[s][0] = v.x;
                    w[s][1] = v.y;
                } else {
#pragma unroll
                    for (int c = 0; c < WORDS / 4; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4*>(src + 16 * c);
                        w[s][4 * c + 0] = v.x;
                        w[s][4 * c + 1] = v.y;
                        w[s][4 * c + 2] = v.z;
                        w[s][4 * c + 3] = v.w;
                    }
                }
            }
        }
        __syncwarp();   // the group's reads before any of its in-place writes
#pragma unroll
        for (int s = 0; s < 2; ++s) {
            const int r = dft_row<G>(g, s, lane);
            const int pair = dft_pair<G>(s, lane);
            const int in_piece = (pair & 3) * 4;
            // the unit's two channels (a: words 0..G/2-1, b: words G/2..G-1) transformed as
            // one packed pair
            fx2 xab[G];
#pragma unroll
            for (int h = 0; h < G / 2; ++h) {
                const uint32_t ua = w[s][h], ub = w[s][G / 2 + h];
                xab[2 * h] = fx2(Io16<T16>::lo(ua), Io16<T16>::lo(ub));
                xab[2 * h + 1] = fx2(Io16<T16>::hi(ua), Io16<T16>::hi(ub));
            }
            fx2 pab[G];
            rdft_planes<G>(xab, pab);
            const int phys = ((pair >> 2) ^ ((r >> 2) & 1)) * 16 + in_piece;   // SWIZZLE_32B
            uint8_t* dst = xs + g * L::SBO + (r & 7) * kRowBytes32 + phys;
#pragma unroll
            for (int p = 0; p < G; ++p)
                *reinterpret_cast<uint32_t*>(dst + L::plane_offset(p)) = Io16<T16>::pack(pab[p].x, pab[p].y);
        }
    }
}

// ------------------------------------------------------------ epilogue role
// Warp (q, half): tokens 32q..32q+31 (TMEM lane quarter q), output channels
// [half*NO/2, (half+1)*NO/2) of the work item, in groups of OG = 32/G channels.
// TMEM is read in batches of EB = 2 groups (G x 2*OG = 64 registers), so a warp waits for
// half as many TMEM loads; the batch's biases are loaded before the wait.
// Per group: inverse real DFT + bias (channel pairs packed as fx2), bf16, one 64-byte row
// per lane into a SWIZZLE_64B staging tile [32 tokens x 32 columns] of the warp's own; a
// batch's EB groups take the warp's EB tiles, then one proxy fence and lane 0's TMA stores
// of all of them under one commit group (so the next batch waits once for the previous
// batch's tiles to be read); the epilogue warps never wait for one another.  Arrives on
// `acc_empty` once its last TMEM load has landed.
template <int G, class T16>
__device__ __forceinline__ void epilogue_tile(const TmParams& p, const CUtensorMap* tmap_y, uint32_t tmem,
                                              int q, int half, int lane, long long n0, int oc, uint8_t* wstage,
                                              int& ybuf, uint32_t acc_empty) {
    using C = Cfg<G>;
    constexpr int OG = C::OG;
    constexpr int EB = 2;                          // groups per TMEM load batch
    static_assert(EB <= kYWarpBufs, "a batch's groups take the warp's staging tiles");
    const int n_groups = (p.NO / 2) / OG;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const long long row0 = n0 + q * 32;            // first token of this warp's rows
    const int swz = (lane >> 1) & 3;               // SWIZZLE_64B of the staging rows
    const uint64_t pol_y = p.l2hint ? ptx::l2_policy_evict_first() : 0ull;
#pragma unroll 1
    for (int g0 = 0; g0 < n_groups; g0 += EB) {
        const int o_loc0 = half * (p.NO / 2) + g0 * OG;
        // biases of the batch's channels (0 past Cout or without bias), before the TMEM wait
        float bv[EB * OG];
#pragma unroll
        for (int j = 0; j < EB * OG; ++j) {
            const int o = oc * p.NO + o_loc0 + j;
            bv[j] = (p.bias != nullptr && o < p.Cout) ? __ldg(p.bias + o) : 0.0f;
        }
        // a batch past the last group reads accumulator columns that are never used
        // (inside the 512 allocated: (G-1)*NO + NO/2 + EB*OG <= 512 for every plan)
        uint32_t r[G][EB * OG];
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_ld_32x32b<EB * OG>(lane_addr + pl * p.NO + o_loc0, r[pl]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_regs_ready<EB * OG>(r[pl]);
        if (g0 + EB >= n_groups) {
            ptx::tc_fence_before();
            ptx::mbar_arrive(acc_empty);           // TMEM no longer needed by this thread
        }
#pragma unroll
        for (int gi = 0; gi < EB; ++gi) {
            if (g0 + gi >= n_groups) break;
            // the lane's staging row: OG channels x G outputs, channel-major, packed in pairs
            uint32_t pk[OG * G / 2];
#pragma unroll
            for (int j = 0; j < OG; j += 2) {
                fx2 z[G], y2[G];
#pragma unroll
                for (int pl = 0; pl < G; ++pl)
                    z[pl] = fx2(__uint_as_float(r[pl][gi * OG + j]), __uint_as_float(r[pl][gi * OG + j + 1]));
                z[0] += fx2(bv[gi * OG + j], bv[gi * OG + j + 1]);
                RealIdft<G, fx2>::run(z, y2);
                if (p.act == kActGelu) {
#pragma unroll
                    for (int gg = 0; gg < G; ++gg) y2[gg] = gelu2(y2[gg]);
                }
#pragma unroll
                for (int gg = 0; gg < G; gg += 2) {
                    pk[(j * G + gg) / 2] = Io16<T16>::pack(y2[gg].x, y2[gg + 1].x);
                    pk[((j + 1) * G + gg) / 2] = Io16<T16>::pack(y2[gg].y, y2[gg + 1].y);
                }
            }
            if (gi == 0) {
                // the previous batch's tiles (one commit group) must have been read
                if (lane == 0) ptx::bulk_wait_group_read<0>();
                __syncwarp();
            }
            uint8_t* rowp = wstage + static_cast<size_t>(gi) * kYWarpBufBytes + lane * (kYCols * 2);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                *reinterpret_cast<uint4*>(rowp + ((k ^ swz) * 16)) =
                    make_uint4(pk[4 * k + 0], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
#pragma unroll
            for (int gi = 0; gi < EB; ++gi) {
                const int o0 = oc * p.NO + o_loc0 + gi * OG;
                // a store only starts inside the tensor; its clipped parts are not written
                if (g0 + gi < n_groups && row0 < p.N && o0 < p.Cout)
                    ptx::tma_store_2d_h(tmap_y, ptx::smem_u32(wstage + static_cast<size_t>(gi) * kYWarpBufBytes),
                                        o0 * G, static_cast<int>(row0), p.l2hint != 0, pol_y);
            }
            ptx::bulk_commit_group();
        }
    }
    (void)ybuf;
}

}  // namespace tm

template <int G, bool STREAM_W, class T16>
__global__ void __launch_bounds__(tm::Cfg<G>::kThreads, 1)
    eqlin_fwd_tm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_y,
                        const TmParams p) {
    using C = tm::Cfg<G>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align_1k(smem_raw);

    constexpr int SL = tm_weight_slots(G);
    const uint32_t wstage_bytes = STREAM_W ? static_cast<uint32_t>(SL * p.NO * kRowBytes32) : 0u;
    const uint32_t stage_bytes = C::XCHUNK_BYTES + wstage_bytes;
    const int NS = p.stages;
    uint8_t* ystage0 = smem + p.w_region_bytes;
    uint8_t* stage0 = ystage0 + tm::kYStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + static_cast<size_t>(NS) * stage_bytes);
    tc::Ctl* ctl = reinterpret_cast<tc::Ctl*>(bars + 3 * NS + 4);

    const uint32_t s_w = ptx::smem_u32(smem);
    const uint32_t s_stage0 = ptx::smem_u32(stage0);
    auto bar_full = [&](int s) { return ptx::smem_u32(bars + s); };
    auto bar_xhat = [&](int s) { return ptx::smem_u32(bars + NS + s); };
    auto bar_empty = [&](int s) { return ptx::smem_u32(bars + 2 * NS + s); };
    const uint32_t bar_acc_full = ptx::smem_u32(bars + 3 * NS + 0);
    const uint32_t bar_acc_empty = ptx::smem_u32(bars + 3 * NS + 1);
    const uint32_t bar_w_full = ptx::smem_u32(bars + 3 * NS + 2);
    const uint32_t bar_drain = ptx::smem_u32(bars + 3 * NS + 3);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(bar_full(s), 1);
            ptx::mbar_init(bar_xhat(s), C::kDftThreads);
            ptx::mbar_init(bar_empty(s), 1);
        }
        ptx::mbar_init(bar_acc_full, 1);
        ptx::mbar_init(bar_acc_empty, tm::kEpiThreads);
        ptx::mbar_init(bar_w_full, 1);
        ptx::mbar_init(bar_drain, 1);
        ctl->abort = 0;
        ptx::fence_mbar_init();
    }
    if (warp == C::kWarpMma) {
        ptx::tmem_alloc(ptx::smem_u32(&ctl->tmem_base), 512);
        ptx::tmem_relinquish();
    }
    if (warp == C::kWarpProducer && lane == 0) {
        ptx::prefetch_tmap(&tmap_x);
        ptx::prefetch_tmap(&tmap_y);
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const bool hint = p.l2hint != 0;
    const uint64_t pol_w = hint ? ptx::l2_policy_evict_last() : 0ull, pol_x = hint ? ptx::l2_policy_evict_first() : 0ull;
    auto load_weights = [&]() {
        ptx::mbar_arrive_expect_tx(bar_w_full, p.w_img_bytes);
        for (uint32_t off = 0; off < p.w_img_bytes; off += 32768u)
            ptx::bulk_load_h(s_w + off, p.w_img + off, min(32768u, p.w_img_bytes - off), bar_w_full, hint, pol_w);
    };
    // weights that no kernel of the stream writes are staged while the previous kernel drains
    if constexpr (!STREAM_W) {
        if (p.w_early && warp == C::kWarpProducer && lane == 0) load_weights();
    }
    // The next forward of the stream may begin launching (its CTAs take an SM as one of
    // ours exits); every access to x and y below waits until the previous kernel of the
    // stream has completed, so y / x aliasing between consecutive calls stays safe.
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();

    if (warp == C::kWarpProducer) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            if constexpr (!STREAM_W) {
                if (!p.w_early) load_weights();
            }
            int stage = 0;
            uint32_t phase = 0;
            long long issued = 0;
            bool ok = true;
            // x chunks of work item wk into L2 (a hint: the loads below still bring them)
            auto prefetch_item = [&](long long wk) {
                if (wk >= p.n_work) return;
                const int n0 = static_cast<int>(wk / p.n_oc) * tm::kM;
                for (int c = 0; c < p.nK; ++c)
#pragma unroll
                    for (int bx = 0; bx < C::X_NBOX; ++bx)
                        ptx::tma_prefetch_l2_2d(&tmap_x, c * C::XROW_ELEMS + bx * C::X_BOX, n0);
            };
            for (int j = 1; j < p.pf; ++j) prefetch_item(blockIdx.x + static_cast<long long>(j) * gridDim.x);
            for (int wk = blockIdx.x; ok && wk < p.n_work; wk += gridDim.x) {
                const int tile = wk / p.n_oc, oc = wk % p.n_oc;
                const int n0 = tile * tm::kM;
                if (p.pf > 0) prefetch_item(wk + static_cast<long long>(p.pf) * gridDim.x);
                for (int c = 0; c < p.nK; ++c) {
                    if (!tc::wait_bounded(bar_empty(stage), phase ^ 1u, ctl, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    // test hook (failure detection): stop issuing after inject_stop chunks, so
                    // the consumers' bounded waits run out; -1 (always, outside tests) = off
                    if (issued == p.inject_stop) {
                        ok = false;
                        break;
                    }
                    const uint32_t dst = s_stage0 + stage * stage_bytes;
                    ptx::mbar_arrive_expect_tx(bar_full(stage), stage_bytes);
#pragma unroll
                    for (int bx = 0; bx < C::X_NBOX; ++bx)
                        ptx::tma_load_2d_h(dst + bx * C::X_BOX_BYTES, &tmap_x, c * C::XROW_ELEMS + bx * C::X_BOX, n0,
                                           bar_full(stage), hint, pol_x);
                    if constexpr (STREAM_W) {
                        ptx::bulk_load_h(dst + C::XCHUNK_BYTES,
                                         p.w_img + static_cast<size_t>(oc * p.nK + c) * wstage_bytes, wstage_bytes,
                                         bar_full(stage), hint, pol_w);
                    }
                    ++issued;
                    if (++stage == NS) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every copy started here lands before the CTA exits (bounded)
            for (int s = 0; s < NS; ++s) {
                const long long times = issued > s ? (issued - s + NS - 1) / NS : 0;
                if (times > 0) {
                    const uint32_t par = static_cast<uint32_t>((times - 1) & 1);
                    const uint64_t t0 = ptx::globaltimer_ns();
                    while (!ptx::mbar_try_wait(bar_full(s), par)) {
                        if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
                            atomicCAS(p.status, 0, kDeviceErrTimeout);
                            break;
                        }
                    }
                }
            }
            if constexpr (!STREAM_W) {
                const uint64_t t0 = ptx::globaltimer_ns();
                while (!ptx::mbar_try_wait(bar_w_full, 0)) {
                    if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
                        atomicCAS(p.status, 0, kDeviceErrTimeout);
                        break;
                    }
                }
            }
        }
    } else if (warp == C::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if constexpr (!STREAM_W) ok = tc::wait_bounded(bar_w_full, 0, ctl, p.status, p.timeout_ns);
            const uint32_t ID = idesc_f16kind_f32(tm::kM, p.NO, Io16<T16>::kUmmaFormat, false, false);
            const uint32_t ID_NEGB = idesc_f16kind_f32(tm::kM, p.NO, Io16<T16>::kUmmaFormat, false, true);
            // complex products: N = 2*NO output columns, the Re and Im planes of D side by side
            const uint32_t ID2 = idesc_f16kind_f32(tm::kM, G > 2 ? 2 * p.NO : p.NO, Io16<T16>::kUmmaFormat, false, false);
            const uint32_t wplane = static_cast<uint32_t>(p.NO) * kRowBytes32;
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int wk = blockIdx.x; ok && wk < p.n_work; wk += gridDim.x, ++it) {
                if (!tc::wait_bounded(bar_acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, ctl, p.status,
                                      p.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                for (int c = 0; c < p.nK; ++c) {
                    if (!tc::wait_bounded(bar_xhat(stage), phase, ctl, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t xb = s_stage0 + stage * stage_bytes;
                    const uint32_t wb = STREAM_W ? xb + C::XCHUNK_BYTES
                                                 : s_w + static_cast<uint32_t>(c * SL) * wplane;
                    const uint32_t a_lo = ptx::sdesc_sw32_lo(xb), b_lo = ptx::sdesc_sw32_lo(wb);
                    const uint32_t wplane16 = wplane >> 4;
                    const uint32_t acc0 = c > 0 ? 1u : 0u;
                    auto A = [&](int pl) {
                        return ptx::sdesc_from_halves(tm::spec_desc_hi<G>(),
                                                      a_lo + tm::SpecLayout<G>::plane_offset(pl) / 16);
                    };
                    auto B = [&](int pl) { return ptx::sdesc_sw32_from_lo(b_lo + static_cast<uint32_t>(pl) * wplane16); };
                    auto D = [&](int pl) { return tmem_base + static_cast<uint32_t>(pl * p.NO); };
                    ptx::umma_f16(D(0), A(0), B(0), ID, acc0);          // k = 0
                    ptx::umma_f16(D(1), A(1), B(1), ID, acc0);          // k = G/2
#pragma unroll
                    for (int k = 1; k < G / 2; ++k) {                   // (Xr + i Xi)(Wr + i Wi)
                        const int pr = 2 * k, pi = 2 * k + 1;
                        if constexpr (tm_pair_slots(G)) {
                            const int s = pair_first_slot(k);
                            ptx::umma_f16(D(pr), A(pr), B(s + 1), ID2, acc0);   // [Dr|Di] += Xr [Wr; Wi]
                            ptx::umma_f16(D(pr), A(pi), B(s), ID2, 1u);         // [Dr|Di] += Xi [-Wi; Wr]
                        } else {
                            ptx::umma_f16(D(pr), A(pr), B(pr), ID2, acc0);      // [Dr|Di] += Xr [Wr; Wi]
                            ptx::umma_f16(D(pr), A(pi), B(pi), ID_NEGB, 1u);    // Dr += Xi (-Wi)
                            ptx::umma_f16(D(pi), A(pi), B(pr), ID, 1u);         // Di += Xi Wr
                        }
                    }
                    ptx::umma_commit(bar_empty(stage));
                    if (++stage == NS) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::umma_commit(bar_acc_full);
            }
            ptx::umma_commit(bar_drain);
            const uint64_t t0 = ptx::globaltimer_ns();
            while (!ptx::mbar_try_wait(bar_drain, 0)) {
                if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
                    atomicCAS(p.status, 0, kDeviceErrTimeout);
                    break;
                }
            }
        }
    } else if (warp >= C::kWarpDft0) {
        // ------------------------------------------------------------ DFT warps
        const int dft_tid = threadIdx.x - C::kWarpDft0 * 32;
        int stage = 0;
        uint32_t phase = 0;
        for (int wk = blockIdx.x; wk < p.n_work; wk += gridDim.x) {
            bool ok = true;
            for (int c = 0; c < p.nK; ++c) {
                const bool got = tc::wait_bounded(bar_full(stage), phase, ctl, p.status, p.timeout_ns);
                if (!ptx::named_bar_and(tm::kBarDft, C::kDftThreads, got)) {
                    ok = false;
                    break;
                }
                tm::dft_chunk<G, T16>(stage0 + static_cast<size_t>(stage) * stage_bytes, dft_tid);
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(bar_xhat(stage));
                if (++stage == NS) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const int half = warp >> 2;
        uint8_t* wstage = ystage0 + static_cast<size_t>(warp) * tm::kYWarpBufs * tm::kYWarpBufBytes;
        int ybuf = 0;
        int it = 0;
        for (int wk = blockIdx.x; wk < p.n_work; wk += gridDim.x, ++it) {
            const bool got = tc::wait_bounded(bar_acc_full, static_cast<uint32_t>(it) & 1u, ctl, p.status,
                                              p.timeout_ns);
            if (!ptx::named_bar_and(tm::kBarEpi, tm::kEpiThreads, got)) break;
            ptx::tc_fence_after();
            const int tile = wk / p.n_oc, oc = wk % p.n_oc;
            tm::epilogue_tile<G, T16>(p, &tmap_y, tmem_base, warp & 3, half, lane,
                                 static_cast<long long>(tile) * tm::kM, oc, wstage, ybuf, bar_acc_empty);
        }
        // the y stores must be complete (not only read) before the CTA exits
        if (lane == 0) ptx::bulk_wait_group<0>();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == C::kWarpMma) {
        __syncwarp();
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace eqlin
