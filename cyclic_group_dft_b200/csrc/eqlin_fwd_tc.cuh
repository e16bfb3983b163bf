// eqlin_fwd_tc.cuh -- fused EQ-Linear forward for 16-bit (bf16 or fp16) I/O on sm_100a.
//
// Operation (page "Flash EQ-Linear: Accelerating Equivariant Linear Layers via
// Group-wise Discrete Fourier Transform", sections "Percepcion Central" and
// "Enfoque Algoritmico"):
//     y[n,o,g] = bias[o] + sum_{i,h} w[o,i,(g-h) mod G] x[n,i,h]
// computed as  X^ = rDFT_G(x)  ->  Y^_k = W^_k X^_k  (k = 0..G/2)  ->  y = irDFT_G(Y^) + bias,
// all in one persistent kernel; nothing is written to global memory between the steps
// (section "Implementacion": fused dataflow, Fourier fragments kept on chip).
//
// Per CTA (one per SM, persistent over work items = (token tile, 128-row output chunk)):
//   warp 12     TMA producer: x chunks [BN tokens x 32 channels x G] (16 KB) into a smem
//               ring (plus the weight chunk when the weights are streamed).
//   warps 8-11  DFT: read a landed x chunk, real DFT over G in fp32 registers, write the
//               spectrum's pair slots [BN x 32] bf16 back IN PLACE in the UMMA K-major
//               SWIZZLE_64B layout (the stage holds the x chunk and, past its end, the
//               spectrum's extra -Im slots).
//   warp 13     MMA issuer (one thread) + TMEM owner: per chunk and frequency,
//               tcgen05.mma with A = W^ plane [128 out-rows x 32], B = X^ plane [BN x 32],
//               D in TMEM (lane = output channel, column = token).  A complex frequency
//               takes two products of N = 2*BN that write its Re and Im planes of D at
//               once: the DFT stores [-Im, Re, Im] of X^ back to back (pair slots,
//               eqlin_layout.h), so B = [Xr; Xi] pairs with Wr and B = [-Xi; Xr] with
//               Wi, and only Re and Im of W^ are stored.  Two accumulators
//               (G*BN = 256 columns each) alternate between work items, so the MMAs of
//               one tile overlap the epilogue of the previous one.
//   warps 0-7   epilogue: tcgen05.ld of all G planes of a token group, inverse real DFT
//               (1/G and 2/G are folded into W^), + bias, round to bf16, write the
//               group's y block [TG tokens x 32*G columns] into the warp's own staging
//               tile (a warp writes 32 consecutive o -> one contiguous 32*G*2-byte run
//               per token) and lane 0 stores it with TMA (rows past N and columns past
//               Cout*G are clipped by the tensor map).  Warps w and w+4 share TMEM lane
//               quarter w and split the tile's tokens.
// All waits are bounded (globaltimer); on expiry the kernel records EQLIN_ERR_TIMEOUT
// in the status word, every role leaves its loop, in-flight copies and MMAs are
// drained with bounded waits, and TMEM is freed before exit.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "eqlin_layout.h"
#include "group_dft.cuh"
#include "io16.cuh"
#include "sm100_ptx.cuh"

namespace eqlin {

struct TcParams {
    const uint8_t* w_img;   // frequency-domain weight image (layout: eqlin_layout.h)
    uint8_t* y;             // [N, Cout, G] output (direct stores, ybufs == 0)
    const float* bias;      // [Cout] fp32, or nullptr
    int* status;            // device status word (first error wins)
    long long N;
    int Cout;
    int nK;                 // 32-channel chunks along Cin
    int rows;               // weight rows per sub-block (resident: Cout rounded to 8; streamed: 128)
    int n_oc;               // 128-row output chunks
    int n_work;             // n_tiles * n_oc
    int stages;             // smem ring depth
    uint32_t w_region_bytes;  // smem reserved for resident weights (0 when streamed)
    uint32_t ystage_bytes;    // y staging per epilogue warp (ybufs buffers of TG x 32*G bf16)
    int ybufs;                // 1 or 2 staging buffers per epilogue warp; 0 = direct stores
    int yq;                   // TMEM lane quarters that hold output rows, each with staging (1..4)
    uint32_t w_img_bytes;     // bytes of the resident image to copy
    unsigned long long timeout_ns;
    long long inject_stop;  // test hook: chunks issued per CTA before the producer stops; -1 = never
    int act;                  // epilogue activation after the bias: kActNone or kActGelu
    // 1: the weights (and bias) were complete before the previous kernel of the stream was
    // launched (a handle's weights: prepare synchronises its stream), so their loads may
    // start before griddepcontrol.wait and overlap the previous kernel's tail.  0: they may
    // be written by the previous kernel of the stream; every load waits.
    int w_early;
    // L2 prefetch distance of the producer, in this CTA's work items: while loading item
    // i it asks the TMA unit to bring item i + pf into L2, so more of x is in flight than
    // the shared-memory ring holds.  0 = off.
    int pf;
    // 1: copies carry L2 eviction priorities: the weights (re-read by every CTA) evict
    // last, x and y (streamed once) evict first.  0: plain copies.
    int l2hint;
};

namespace tc {

constexpr int kThreads = 448;
constexpr int kEpiWarps = 8;
constexpr int kEpiThreads = kEpiWarps * 32;
constexpr int kWarpDft0 = 8;
constexpr int kWarpProducer = 12;
constexpr int kWarpMma = 13;
constexpr int kBarDft = 1;   // named barrier ids (0 is __syncthreads)
constexpr int kBarEpi = 2;
constexpr int kYBoxCols2 = 256;  // widest y TMA store box (bf16 columns)

// NACC accumulator buffers of G*BN TMEM columns each share the 512 columns: with two,
// the MMAs of one tile overlap the epilogue of the previous one; with one, each MMA
// covers twice the tokens (half the weight-operand traffic and MMA count per token).
template <int G, int NACC = 2>
struct Shape {
    static constexpr int kNumAcc = NACC;
    static constexpr int BN = (512 / (G * NACC)) < 128 ? (512 / (G * NACC)) : 128;  // tokens per tile (MMA N)
    static constexpr int PLANE_BYTES = BN * kPlaneRowBytes;          // one frequency plane
    static constexpr int XCHUNK_BYTES = G * PLANE_BYTES;             // == BN * 32 * G * 2 (the x chunk)
    static constexpr int SLOTS = pair_slots(G);                      // spectrum slots (eqlin_layout.h)
    static constexpr int SPEC_BYTES = SLOTS * PLANE_BYTES;           // the chunk's spectrum, in place
    static constexpr int XROW_ELEMS = kChunkK * G;                   // one token row of a chunk
    static constexpr int BOX_ELEMS = XROW_ELEMS < 256 ? XROW_ELEMS : 256;
    static constexpr int NBOX = XROW_ELEMS / BOX_ELEMS;
    static constexpr int WSTAGE_BYTES = G * kMmaM * kPlaneRowBytes;  // streamed weight chunk
    static constexpr int ACC_COLS = G * BN;                          // one accumulator
    static constexpr int TMEM_COLS = 512;
    static constexpr int TG = (64 / G) < BN / 2 ? (64 / G) : BN / 2;  // tokens per epilogue group
    static_assert(XCHUNK_BYTES % 1024 == 0 && SPEC_BYTES % 1024 == 0, "stage alignment");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N");
    static_assert(NACC * ACC_COLS <= TMEM_COLS, "TMEM columns");
    static_assert((BN / 2) % TG == 0, "epilogue groups");
};

// suspend-time hint of a waiting thread (it wakes as soon as the phase completes)
constexpr uint32_t kWaitSleepNs = 20000;

struct Ctl {
    volatile int abort;
    uint32_t tmem_base;
};

// Bounded mbarrier wait.  Returns false (after flagging) on timeout or abort.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, Ctl* ctl,
                                             int* status, unsigned long long timeout_ns) {
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

// Bounded wait that ignores the abort flag, for copies or MMAs in flight before exit.
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

// ---------------------------------------------------------------- DFT role
// 128 threads.  Unit = one token row x two adjacent channels (2*G bf16).
// Lanes 0-15 take row r, lanes 16-31 row r+1; lane&15 selects the channel pair.
template <int G, int NACC, class T16>
__device__ __forceinline__ void dft_chunk(uint8_t* xs, int dft_tid) {
    using S = Shape<G, NACC>;
    constexpr int WORDS = G;                         // 32-bit words per unit (2 ch x G x 2 B / 4)
    constexpr int STEPS = S::BN / 8;                 // 2 rows per step, 4 warps
    const int warp = dft_tid >> 5, lane = dft_tid & 31;
    const int pair = lane & 15;
    const int row0 = warp * (S::BN / 4) + (lane >> 4);
    // element offset of the unit inside a token row, and the TMA box it lives in
    constexpr int UNIT_ELEMS = 2 * G;
    const int e = pair * UNIT_ELEMS;
    const int box = e / S::BOX_ELEMS;
    const int e_in = e % S::BOX_ELEMS;
    const uint8_t* src0 = xs + box * (S::BN * S::BOX_ELEMS * 2) + e_in * 2;

    uint32_t w[STEPS][WORDS];
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int r = row0 + 2 * s;
        const uint8_t* src = src0 + r * (S::BOX_ELEMS * 2);
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
    // every read of this chunk happens before any in-place write
    ptx::named_bar_sync(kBarDft, 128);

    const int chunk = pair >> 2;              // 16-B chunk of the 64-B plane row
    const int in_chunk = (pair & 3) * 4;      // byte inside it
#pragma unroll
    for (int s = 0; s < STEPS; ++s) {
        const int r = row0 + 2 * s;
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
        const int phys = (chunk ^ ((r >> 1) & 3)) * 16 + in_chunk;   // SWIZZLE_64B
        uint8_t* dst = xs + r * kPlaneRowBytes + phys;
        // pair slots: planes 0 and 1, then [-Im, Re, Im] per complex frequency; the sign
        // flip of the packed pair is exact (rounding to nearest even is symmetric)
        *reinterpret_cast<uint32_t*>(dst) = Io16<T16>::pack(pab[0].x, pab[0].y);
        *reinterpret_cast<uint32_t*>(dst + S::PLANE_BYTES) = Io16<T16>::pack(pab[1].x, pab[1].y);
#pragma unroll
        for (int k = 1; k < G / 2; ++k) {
            const uint32_t re = Io16<T16>::pack(pab[2 * k].x, pab[2 * k].y);
            const uint32_t im = Io16<T16>::pack(pab[2 * k + 1].x, pab[2 * k + 1].y);
            uint8_t* d = dst + pair_first_slot(k) * S::PLANE_BYTES;
            *reinterpret_cast<uint32_t*>(d) = im ^ 0x80008000u;
            *reinterpret_cast<uint32_t*>(d + S::PLANE_BYTES) = re;
            *reinterpret_cast<uint32_t*>(d + 2 * S::PLANE_BYTES) = im;
        }
    }
}

// ------------------------------------------------------------ epilogue role
// Warp (q, half): TMEM lane quarter q (output rows 32q..32q+31 of the chunk), tokens
// [half*BN/2, (half+1)*BN/2) of the tile held in accumulator `acc` (column base).
// The warp reads a group of TG tokens x its 32 output channels (32*G columns) from
// TMEM, stages it in its own buffer and lane 0 stores it with TMA, so the epilogue
// warps never wait for one another.  `wstage`: this warp's p.ybufs buffers; `ybuf`
// alternates.
template <int G, int NACC, class T16>
__device__ __forceinline__ void epilogue_tile(const TcParams& p, const CUtensorMap* tmap_y, uint32_t acc,
                                              int q, int half, int lane, long long n0, int oc, uint8_t* wstage,
                                              int& ybuf) {
    using S = Shape<G, NACC>;
    constexpr int TG = S::TG;
    constexpr int WCOLS = 32 * G;                           // y columns of the warp's 32 outputs
    constexpr int YBC = WCOLS < kYBoxCols2 ? WCOLS : kYBoxCols2;  // TMA box columns
    constexpr int NYB = WCOLS / YBC;
    constexpr int BOX_BYTES = TG * YBC * 2;
    const int o_local = q * 32 + lane;
    const int o = oc * kMmaM + o_local;
    const bool valid_o = o < p.Cout;
    const float b = (p.bias != nullptr && valid_o) ? p.bias[o] : 0.0f;
    const uint32_t lane_addr = acc + (static_cast<uint32_t>(q * 32) << 16);
    const int t0 = half * (S::BN / 2);
    const int col = lane * G;                               // first staged column of this lane
    const uint64_t pol_y = p.l2hint ? ptx::l2_policy_evict_first() : 0ull;
    uint8_t* lane_off0 = wstage + (col / YBC) * BOX_BYTES + (col % YBC) * 2;
#pragma unroll 1
    for (int j = 0; j < S::BN / 2 / TG; ++j) {
        uint32_t r[G][TG];
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_ld_32x32b<TG>(lane_addr + pl * S::BN + t0 + j * TG, r[pl]);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int pl = 0; pl < G; ++pl) ptx::tmem_regs_ready<TG>(r[pl]);
        if (p.ybufs == 0) {
            // direct stores: lane o writes its G outputs (2G bytes) of each token, so a warp
            // writes 32 consecutive channels = one contiguous 64G-byte run per token
            const long long row0 = n0 + t0 + j * TG;
            if (valid_o) {
#pragma unroll
                for (int t = 0; t < TG; ++t) {
                    if (row0 + t >= p.N) break;
                    float z[G], yv[G];
#pragma unroll
                    for (int pl = 0; pl < G; ++pl) z[pl] = __uint_as_float(r[pl][t]);
                    z[0] += b;
                    RealIdft<G>::run(z, yv);
                    if (p.act == kActGelu) {
#pragma unroll
                        for (int g = 0; g < G; g += 2) {
                            const fx2 u = gelu2(fx2(yv[g], yv[g + 1]));
                            yv[g] = u.x;
                            yv[g + 1] = u.y;
                        }
                    }
                    uint8_t* dst = p.y + ((row0 + t) * p.Cout + o) * (2 * G);
                    if constexpr (G == 2) {
                        *reinterpret_cast<uint32_t*>(dst) = Io16<T16>::pack(yv[0], yv[1]);
                    } else if constexpr (G == 4) {
                        *reinterpret_cast<uint2*>(dst) =
                            make_uint2(Io16<T16>::pack(yv[0], yv[1]), Io16<T16>::pack(yv[2], yv[3]));
                    } else {
#pragma unroll
                        for (int c = 0; c < G / 8; ++c) {
                            *reinterpret_cast<uint4*>(dst + 16 * c) = make_uint4(
                                Io16<T16>::pack(yv[8 * c + 0], yv[8 * c + 1]), Io16<T16>::pack(yv[8 * c + 2], yv[8 * c + 3]),
                                Io16<T16>::pack(yv[8 * c + 4], yv[8 * c + 5]), Io16<T16>::pack(yv[8 * c + 6], yv[8 * c + 7]));
                        }
                    }
                }
            }
            continue;
        }
        // the buffer about to be written was stored p.ybufs groups ago: wait until read
        if (lane == 0) {
            if (p.ybufs == 2) ptx::bulk_wait_group_read<1>();
            else ptx::bulk_wait_group_read<0>();
        }
        __syncwarp();
        uint8_t* lane_off = lane_off0 + static_cast<size_t>(ybuf) * (NYB * BOX_BYTES);
        if (valid_o) {
#pragma unroll
            for (int t = 0; t < TG; ++t) {
                float z[G], yv[G];
#pragma unroll
                for (int pl = 0; pl < G; ++pl) z[pl] = __uint_as_float(r[pl][t]);
                z[0] += b;  // the DC term appears with weight 1 in every output
                RealIdft<G>::run(z, yv);
                if (p.act == kActGelu) {
#pragma unroll
                    for (int g = 0; g < G; g += 2) {
                        const fx2 u = gelu2(fx2(yv[g], yv[g + 1]));
                        yv[g] = u.x;
                        yv[g + 1] = u.y;
                    }
                }
                uint8_t* dst = lane_off + t * (YBC * 2);
                if constexpr (G == 2) {
                    *reinterpret_cast<uint32_t*>(dst) = Io16<T16>::pack(yv[0], yv[1]);
                } else if constexpr (G == 4) {
                    *reinterpret_cast<uint2*>(dst) =
                        make_uint2(Io16<T16>::pack(yv[0], yv[1]), Io16<T16>::pack(yv[2], yv[3]));
                } else {
#pragma unroll
                    for (int c = 0; c < G / 8; ++c) {
                        *reinterpret_cast<uint4*>(dst + 16 * c) = make_uint4(
                            Io16<T16>::pack(yv[8 * c + 0], yv[8 * c + 1]), Io16<T16>::pack(yv[8 * c + 2], yv[8 * c + 3]),
                            Io16<T16>::pack(yv[8 * c + 4], yv[8 * c + 5]), Io16<T16>::pack(yv[8 * c + 6], yv[8 * c + 7]));
                    }
                }
            }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            // every store starts inside the tensor: rows past N and columns past Cout*G
            // of a started box are clipped, boxes that would start outside are skipped
            const long long row = n0 + t0 + j * TG;
            if (row < p.N) {
                const uint32_t src = ptx::smem_u32(wstage + static_cast<size_t>(ybuf) * (NYB * BOX_BYTES));
#pragma unroll
                for (int bx = 0; bx < NYB; ++bx) {
                    const int o_first = oc * kMmaM + q * 32 + bx * (YBC / G);
                    if (o_first < p.Cout)
                        ptx::tma_store_2d_h(tmap_y, src + bx * BOX_BYTES, o_first * G, static_cast<int>(row),
                                            p.l2hint != 0, pol_y);
                }
            }
            ptx::bulk_commit_group();
        }
        if (p.ybufs == 2) ybuf ^= 1;
    }
}

}  // namespace tc

template <int G, bool STREAM_W, int NACC, class T16>
__global__ void __launch_bounds__(tc::kThreads, 1)
    eqlin_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_y,
                        const TcParams p) {
    using S = tc::Shape<G, NACC>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = ptx::smem_align_1k(smem_raw);

    // a stage: the x chunk, transformed in place into its (larger) spectrum, then the
    // streamed weight chunk; the copies fill the x chunk and the weight chunk
    constexpr uint32_t STAGE_BYTES = S::SPEC_BYTES + (STREAM_W ? S::WSTAGE_BYTES : 0);
    constexpr uint32_t STAGE_TX = S::XCHUNK_BYTES + (STREAM_W ? S::WSTAGE_BYTES : 0);
    const int NS = p.stages;
    uint8_t* ystage0 = smem + p.w_region_bytes;   // y staging, one area per active epilogue warp
    uint8_t* stage0 = ystage0 + 2 * static_cast<size_t>(p.yq) * p.ystage_bytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(stage0 + static_cast<size_t>(NS) * STAGE_BYTES);
    tc::Ctl* ctl = reinterpret_cast<tc::Ctl*>(bars + 3 * NS + 2 * NACC + 2);

    const uint32_t s_w = ptx::smem_u32(smem);
    const uint32_t s_stage0 = ptx::smem_u32(stage0);
    auto bar_full = [&](int s) { return ptx::smem_u32(bars + s); };
    auto bar_xhat = [&](int s) { return ptx::smem_u32(bars + NS + s); };
    auto bar_empty = [&](int s) { return ptx::smem_u32(bars + 2 * NS + s); };
    auto bar_acc_full = [&](int a) { return ptx::smem_u32(bars + 3 * NS + a); };
    auto bar_acc_empty = [&](int a) { return ptx::smem_u32(bars + 3 * NS + NACC + a); };
    const uint32_t bar_w_full = ptx::smem_u32(bars + 3 * NS + 2 * NACC);
    const uint32_t bar_drain = ptx::smem_u32(bars + 3 * NS + 2 * NACC + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            ptx::mbar_init(bar_full(s), 1);
            ptx::mbar_init(bar_xhat(s), 128);
            ptx::mbar_init(bar_empty(s), 1);
        }
        for (int a = 0; a < NACC; ++a) {
            ptx::mbar_init(bar_acc_full(a), 1);
            ptx::mbar_init(bar_acc_empty(a), tc::kEpiThreads);
        }
        ptx::mbar_init(bar_w_full, 1);
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
    // resident weights: one bulk copy per 32 KB, completing on bar_w_full
    auto load_weights = [&]() {
        ptx::mbar_arrive_expect_tx(bar_w_full, p.w_img_bytes);
        for (uint32_t off = 0; off < p.w_img_bytes; off += 32768u) {
            const uint32_t n = min(32768u, p.w_img_bytes - off);
            ptx::bulk_load_h(s_w + off, p.w_img + off, n, bar_w_full, hint, pol_w);
        }
    };
    // weights that no kernel of the stream writes are staged while the previous kernel drains
    if constexpr (!STREAM_W) {
        if (p.w_early && warp == tc::kWarpProducer && lane == 0) load_weights();
    }
    // The next forward of the stream may begin launching (its CTAs take an SM as one of
    // ours exits); every access to x and y below waits until the previous kernel of the
    // stream has completed, so y / x aliasing between consecutive calls stays safe.
    ptx::grid_launch_dependents();
    ptx::grid_dependency_wait();

    if (warp == tc::kWarpProducer) {
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
                const int n0 = static_cast<int>(wk / p.n_oc) * S::BN;
                for (int c = 0; c < p.nK; ++c)
#pragma unroll
                    for (int bx = 0; bx < S::NBOX; ++bx)
                        ptx::tma_prefetch_l2_2d(&tmap_x, c * S::XROW_ELEMS + bx * S::BOX_ELEMS, n0);
            };
            for (int j = 1; j < p.pf; ++j) prefetch_item(blockIdx.x + static_cast<long long>(j) * gridDim.x);
            for (int wk = blockIdx.x; ok && wk < p.n_work; wk += gridDim.x) {
                const int tile = wk / p.n_oc, oc = wk % p.n_oc;
                const int n0 = tile * S::BN;
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
                    const uint32_t dst = s_stage0 + stage * STAGE_BYTES;
                    ptx::mbar_arrive_expect_tx(bar_full(stage), STAGE_TX);
#pragma unroll
                    for (int bx = 0; bx < S::NBOX; ++bx) {
                        ptx::tma_load_2d_h(dst + bx * (S::BN * S::BOX_ELEMS * 2), &tmap_x,
                                           c * S::XROW_ELEMS + bx * S::BOX_ELEMS, n0, bar_full(stage), hint, pol_x);
                    }
                    if constexpr (STREAM_W) {
                        ptx::bulk_load_h(dst + S::SPEC_BYTES,
                                         p.w_img + static_cast<size_t>(oc * p.nK + c) * S::WSTAGE_BYTES,
                                         S::WSTAGE_BYTES, bar_full(stage), hint, pol_w);
                    }
                    ++issued;
                    if (++stage == NS) { stage = 0; phase ^= 1u; }
                }
            }
            // drain: every copy this thread started must land before the CTA exits
            for (int s = 0; s < NS; ++s) {
                const long long times = issued > s ? (issued - s + NS - 1) / NS : 0;
                if (times > 0) {
                    const uint32_t par = static_cast<uint32_t>((times - 1) & 1);
                    // bounded, and deliberately blind to the abort flag: a copy in
                    // flight must land before its shared memory is released
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
    } else if (warp == tc::kWarpMma) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if constexpr (!STREAM_W) ok = tc::wait_bounded(bar_w_full, 0, ctl, p.status, p.timeout_ns);
            constexpr uint32_t ID = idesc_f16kind_f32(kMmaM, S::BN, Io16<T16>::kUmmaFormat, false);
            // complex products: N = 2*BN, the Re and Im planes of D side by side
            constexpr uint32_t ID2 = idesc_f16kind_f32(kMmaM, G > 2 ? 2 * S::BN : S::BN, Io16<T16>::kUmmaFormat, false);
            int stage = 0;
            uint32_t phase = 0;
            int it = 0;
            for (int wk = blockIdx.x; ok && wk < p.n_work; wk += gridDim.x, ++it) {
                const int abuf = it % NACC;
                const uint32_t acc_phase = static_cast<uint32_t>(it / NACC) & 1u;
                if (!tc::wait_bounded(bar_acc_empty(abuf), acc_phase ^ 1u, ctl, p.status, p.timeout_ns)) {
                    ok = false;
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t acc_base = tmem_base + static_cast<uint32_t>(abuf * S::ACC_COLS);
                for (int c = 0; c < p.nK; ++c) {
                    if (!tc::wait_bounded(bar_xhat(stage), phase, ctl, p.status, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    const uint32_t xb = s_stage0 + stage * STAGE_BYTES;
                    uint32_t wb, wsub;
                    if constexpr (STREAM_W) {
                        wb = xb + S::SPEC_BYTES;
                        wsub = kMmaM * kPlaneRowBytes;
                    } else {
                        wsub = static_cast<uint32_t>(p.rows) * kPlaneRowBytes;
                        wb = s_w + static_cast<uint32_t>(c * G) * wsub;
                    }
                    // descriptors differ only in their start-address field: build each
                    // one as (constant high half, low half + byte offset / 16)
                    const uint32_t a_lo = ptx::sdesc_sw64_lo(wb), b_lo = ptx::sdesc_sw64_lo(xb);
                    const uint32_t wsub16 = wsub >> 4;
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
                        // real frequencies k = 0 and k = G/2
                        ptx::umma_f16(D(0), A(0), B(0), ID, acc0);
                        ptx::umma_f16(D(1), A(1), B(1), ID, acc0);
                        // complex frequencies: (Wr + i Wi)(Xr + i Xi), two products of N = 2*BN
#pragma unroll
                        for (int k = 1; k < G / 2; ++k) {
                            const int pr = 2 * k, pi = 2 * k + 1, s = pair_first_slot(k);
                            ptx::umma_f16(D(pr), A(pr), B(s + 1), ID2, acc0);   // [Dr|Di] += Wr [Xr; Xi]
                            ptx::umma_f16(D(pr), A(pi), B(s), ID2, 1u);         // [Dr|Di] += Wi [-Xi; Xr]
                        }
                    }
                    ptx::umma_commit(bar_empty(stage));   // stage reusable once these finish
                    if (++stage == NS) { stage = 0; phase ^= 1u; }
                }
                if (!ok) break;
                ptx::umma_commit(bar_acc_full(abuf));
            }
            // drain: all MMAs done before TMEM is released
            ptx::umma_commit(bar_drain);
            const uint64_t t0 = ptx::globaltimer_ns();
            while (!ptx::mbar_try_wait(bar_drain, 0)) {
                if (ptx::globaltimer_ns() - t0 > p.timeout_ns) {
                    atomicCAS(p.status, 0, kDeviceErrTimeout);
                    break;
                }
            }
        }
    } else if (warp >= tc::kWarpDft0) {
        // ------------------------------------------------------------ DFT warps
        const int dft_tid = threadIdx.x - tc::kWarpDft0 * 32;
        int stage = 0;
        uint32_t phase = 0;
        for (int wk = blockIdx.x; wk < p.n_work; wk += gridDim.x) {
            bool ok = true;
            for (int c = 0; c < p.nK; ++c) {
                const bool got = tc::wait_bounded(bar_full(stage), phase, ctl, p.status, p.timeout_ns);
                if (!ptx::named_bar_and(tc::kBarDft, 128, got)) {
                    ok = false;
                    break;
                }
                tc::dft_chunk<G, NACC, T16>(stage0 + static_cast<size_t>(stage) * STAGE_BYTES, dft_tid);
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(bar_xhat(stage));
                if (++stage == NS) { stage = 0; phase ^= 1u; }
            }
            if (!ok) break;
        }
    } else {
        // ------------------------------------------------------------ epilogue warps
        const int half = warp >> 2, q = warp & 3;
        // staging areas exist only for the p.yq lane quarters that hold output rows
        uint8_t* wstage = ystage0 + static_cast<size_t>(half * p.yq + (q < p.yq ? q : 0)) * p.ystage_bytes;
        int ybuf = 0;
        int it = 0;
        for (int wk = blockIdx.x; wk < p.n_work; wk += gridDim.x, ++it) {
            const int abuf = it % NACC;
            const uint32_t acc_phase = static_cast<uint32_t>(it / NACC) & 1u;
            const bool got = tc::wait_bounded(bar_acc_full(abuf), acc_phase, ctl, p.status, p.timeout_ns);
            if (!ptx::named_bar_and(tc::kBarEpi, tc::kEpiThreads, got)) break;
            ptx::tc_fence_after();
            const int tile = wk / p.n_oc, oc = wk % p.n_oc;
            // warps whose lane quarter holds no valid output row skip the work
            if (q < p.yq && oc * kMmaM + q * 32 < p.Cout) {
                const uint32_t acc = tmem_base + static_cast<uint32_t>(abuf * S::ACC_COLS);
                const long long n0 = static_cast<long long>(tile) * S::BN;
                tc::epilogue_tile<G, NACC, T16>(p, &tmap_y, acc, q, half, lane, n0, oc, wstage, ybuf);
            }
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar_acc_empty(abuf));
        }
        // the y stores must be complete (not only read) before the CTA exits
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
