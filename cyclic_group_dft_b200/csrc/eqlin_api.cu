// eqlin_api.cu -- host side of the C ABI declared in include/eqlin.h: argument
// validation, kernel planning (shared-memory budget, ring depth, kernel variant),
// ownership of the frequency-domain weights, TMA descriptor encoding and launches.
#include "eqlin.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "eqlin_bwd_dw.cuh"
#include "eqlin_fwd_tc.cuh"
#include "eqlin_fwd_tcr.cuh"
#include "eqlin_fwd_tm.cuh"
#include "eqlin_layout.h"
#include "eqlin_prep.cuh"

using eqlin::TcParams;
using eqlin::TmParams;

namespace {

constexpr size_t kB200SmemOptin = 232448;   // 227 KB opt-in shared memory per CTA on sm_100
constexpr int kB200SmCount = 148;           // SMs of a B200 (host-only planning queries)
constexpr size_t kSmemAlignSlack = 1024;    // the kernels round their smem base up to 1 KB
constexpr size_t kSmemCtlBytes = 512;       // mbarriers + control block
constexpr int kMaxStages = 12;
constexpr int64_t kMaxChannels = 1 << 16;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

// Kernel variants (EQLIN_ATTR_PATH):
//   0/1  tcgen05, tokens on the MMA N dimension, weights resident / streamed
//   2    fp32 I/O, float64 CUDA-core kernel
//   3/4  tcgen05, tokens on the MMA M dimension, weights resident / streamed
//   5    tcgen05, tokens on N, input spectrum resident across output chunks, weights streamed
enum Path {
    kPathResident = 0,
    kPathStreamed = 1,
    kPathF32 = 2,
    kPathTmResident = 3,
    kPathTmStreamed = 4,
    kPathTnResidentX = 5
};

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(EQLIN_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

struct Plan {
    int io = EQLIN_BF16; // element type of x and y (EQLIN_BF16, EQLIN_F16 or EQLIN_F32)
    int path = kPathF32;
    int nacc = 2;        // TMEM accumulator buffers (tokens-on-N kernel)
    int nK = 0;          // input-channel chunks
    int rows = 0;        // weight rows per image sub-block (tokens-on-M: NO, the MMA N)
    int n_oc = 0;        // output chunks
    int BN = 0;          // tokens per work item
    int stages = 0;
    int TG = 0;          // y TMA store box rows (tokens-on-N)
    int ybufs = 0;       // y staging buffers per epilogue warp (tokens-on-N)
    int box_elems = 0;   // x TMA box columns
    bool x_swizzle128 = false;  // x boxes land SWIZZLE_128B (tokens-on-M, G >= 8)
    uint32_t w_region_bytes = 0, w_img_bytes = 0, ystage_bytes = 0;
    size_t smem_bytes = 0;
    size_t img_alloc_bytes = 0;
    bool tm() const { return path == kPathTmResident || path == kPathTmStreamed; }
    bool tnr() const { return path == kPathTnResidentX; }
    bool streamed() const { return path == kPathStreamed || path == kPathTmStreamed || path == kPathTnResidentX; }
};

// ----------------------------------------------------------------- planning
// Tuning overrides read from the environment: EQLIN_MAX_STAGES caps the ring depth,
// EQLIN_YBUFS (1 or 2) fixes the tokens-on-N y staging depth.
int env_int(const char* name, int dflt) {
    const char* e = std::getenv(name);
    if (!e || !*e) return dflt;
    const int v = std::atoi(e);
    return v > 0 ? v : dflt;
}

// How the tokens-on-N epilogue writes y: staged in shared memory for TMA stores, or with
// plain coalesced stores from registers (a warp writes 32 consecutive channels of a
// token).  Measured on B200: staging wins where the output dominates (p4 C96: 62.1 vs
// 82.8 us); direct stores win where the freed staging space deepens a ring that limits
// the kernel: many input chunks per work item, or the resident-input kernel's weight ring
// (192 -> 768: 174 vs 210 us with 3 instead of 2 weight stages).
// EQLIN_YSTORE=tma|direct overrides.
bool y_direct(bool dflt) {
    const char* e = std::getenv("EQLIN_YSTORE");
    if (e && std::strcmp(e, "direct") == 0) return true;
    if (e && std::strcmp(e, "tma") == 0) return false;
    return dflt;
}

template <int G, int NACC>
int plan_tn_g(int64_t Cout, int64_t Cin, size_t max_smem, Plan* pl) {
    const int max_stages = std::min(kMaxStages, env_int("EQLIN_MAX_STAGES", kMaxStages));
    const int ybufs_env = env_int("EQLIN_YBUFS", 0);
    using S = eqlin::tc::Shape<G, NACC>;
    pl->nacc = NACC;
    pl->nK = static_cast<int>((Cin + eqlin::kChunkK - 1) / eqlin::kChunkK);
    // direct stores from 8 input chunks on (B200: 256 -> 64 at p4, 126.5 vs 139.4 us;
    // 384 -> 96, 189.4 vs 206.1 us), staged TMA stores below (96 -> 96: 62.1 vs 82.8 us)
    const bool direct = y_direct(pl->nK >= 8);
    pl->n_oc = static_cast<int>((Cout + eqlin::kMmaM - 1) / eqlin::kMmaM);
    pl->BN = S::BN;
    pl->TG = S::TG;
    pl->box_elems = S::BOX_ELEMS;
    // y staging: per epilogue warp, ybufs buffers of TG rows x 32*G bf16 columns (4 KB);
    // double-buffered when at least 4 ring stages still fit
    const size_t ybuf = static_cast<size_t>(S::TG) * 32 * G * 2;
    auto fixed_for = [&](int nb) {
        return kSmemAlignSlack + kSmemCtlBytes + static_cast<size_t>(eqlin::tc::kEpiWarps) * nb * ybuf;
    };
    pl->ybufs = 2;
    for (int nb = direct ? 0 : 2; nb >= (direct ? 0 : 1); --nb) {
        if (!direct && ybufs_env && nb != ybufs_env) continue;
        const size_t fixed = fixed_for(nb);
        pl->ybufs = nb;
        pl->ystage_bytes = static_cast<uint32_t>(nb * ybuf);
        if (pl->n_oc == 1) {
            // weights resident in shared memory for the whole kernel
            const int rows = static_cast<int>((Cout + 7) / 8 * 8);
            const size_t img = static_cast<size_t>(G) * pl->nK * rows * eqlin::kPlaneRowBytes;
            // the A operand always reads 128 rows: keep the overrun of the last block inside
            const size_t region = (img + static_cast<size_t>(eqlin::kMmaM - rows) * eqlin::kPlaneRowBytes +
                                   1023) / 1024 * 1024;
            if (max_smem > fixed + region) {
                const size_t stages =
                    std::min<size_t>(max_stages, (max_smem - fixed - region) / S::SPEC_BYTES);
                if (stages >= static_cast<size_t>(nb == 2 && !ybufs_env ? 4 : 2)) {
                    pl->path = kPathResident;
                    pl->rows = rows;
                    pl->stages = static_cast<int>(stages);
                    pl->w_region_bytes = static_cast<uint32_t>(region);
                    pl->w_img_bytes = static_cast<uint32_t>(img);
                    pl->img_alloc_bytes = img;
                    pl->smem_bytes = fixed + region + stages * S::SPEC_BYTES;
                    return EQLIN_OK;
                }
            }
        }
        // weights streamed chunk by chunk next to each x chunk
        if (pl->n_oc > 1 || nb <= 1) {
            const size_t stage = static_cast<size_t>(S::SPEC_BYTES) + S::WSTAGE_BYTES;
            const size_t stages = max_smem > fixed ? std::min<size_t>(max_stages, (max_smem - fixed) / stage) : 0;
            if (stages >= static_cast<size_t>(nb == 2 && !ybufs_env ? 3 : 1)) {
                pl->path = kPathStreamed;
                pl->rows = eqlin::kMmaM;
                pl->stages = static_cast<int>(stages);
                pl->w_region_bytes = 0;
                pl->w_img_bytes = 0;
                pl->img_alloc_bytes = static_cast<size_t>(pl->n_oc) * pl->nK * S::WSTAGE_BYTES;
                pl->smem_bytes = fixed + stages * stage;
                return EQLIN_OK;
            }
        }
    }
    return fail(EQLIN_ERR_UNSUPPORTED, "shape does not fit in shared memory");
}

// Tokens on N with the input spectrum resident: all nK x chunks of a token tile stay in
// smem while the weight chunks of every output chunk stream through a ring.  Applies
// when Cout > 128 (several output chunks) and the slots fit with >= 2 ring stages.
// By default only from 4 input chunks on: below that, re-transforming x per output chunk
// costs less than the resident form's narrower ring (B200, p4: 96 -> 384, 186.5 us
// streamed vs 193.5 us; 64 -> 256, 115.7 vs 122.7 us; 128 -> 512, 314.1 vs 290.8 us).
template <int G>
int plan_tnr_g(int64_t Cout, int64_t Cin, size_t max_smem, bool forced, Plan* pl) {
    using S = eqlin::tc::Shape<G, 2>;
    const int max_stages = std::min(kMaxStages, env_int("EQLIN_MAX_STAGES", kMaxStages));
    const int nK = static_cast<int>((Cin + eqlin::kChunkK - 1) / eqlin::kChunkK);
    const int n_oc = static_cast<int>((Cout + eqlin::kMmaM - 1) / eqlin::kMmaM);
    if (n_oc < 2 || nK > eqlin::tcr::kMaxK || (!forced && nK < 4)) return EQLIN_ERR_UNSUPPORTED;
    const size_t ybuf = static_cast<size_t>(S::TG) * 32 * G * 2;
    // (staging buffers, least ring stages) in order of preference: staged TMA stores with
    // a ring of >= 3 weight chunks, else direct stores (no staging) with >= 2, else one
    // staging buffer with 2; EQLIN_YSTORE=tma|direct keeps to one store mode
    const char* ys = std::getenv("EQLIN_YSTORE");
    const bool only_direct = ys && std::strcmp(ys, "direct") == 0;
    const bool only_tma = ys && std::strcmp(ys, "tma") == 0;
    const int options[5][2] = {{2, 3}, {1, 3}, {0, 2}, {1, 2}, {2, 2}};
    for (const auto& opt : options) {
        const int nb = opt[0];
        if ((only_direct && nb != 0) || (only_tma && nb == 0)) continue;
        const size_t fixed = kSmemAlignSlack + kSmemCtlBytes + static_cast<size_t>(eqlin::tc::kEpiWarps) * nb * ybuf +
                             static_cast<size_t>(nK) * S::SPEC_BYTES;
        if (max_smem <= fixed) continue;
        const size_t stages = std::min<size_t>(max_stages, (max_smem - fixed) / S::WSTAGE_BYTES);
        if (stages < static_cast<size_t>(opt[1])) continue;
        pl->path = kPathTnResidentX;
        pl->nacc = 2;
        pl->nK = nK;
        pl->n_oc = n_oc;
        pl->BN = S::BN;
        pl->TG = S::TG;
        pl->box_elems = S::BOX_ELEMS;
        pl->ybufs = nb;
        pl->ystage_bytes = static_cast<uint32_t>(nb * ybuf);
        pl->rows = eqlin::kMmaM;
        pl->stages = static_cast<int>(stages);
        pl->w_region_bytes = 0;
        pl->w_img_bytes = 0;
        pl->img_alloc_bytes = static_cast<size_t>(n_oc) * nK * S::WSTAGE_BYTES;
        pl->smem_bytes = fixed + stages * S::WSTAGE_BYTES;
        return EQLIN_OK;
    }
    return EQLIN_ERR_UNSUPPORTED;
}

template <int G>
int plan_tm_g(int64_t Cout, int64_t Cin, size_t max_smem, Plan* pl) {
    using C = eqlin::tm::Cfg<G>;
    const int kMaxStages = std::min(::kMaxStages, env_int("EQLIN_MAX_STAGES", ::kMaxStages));
    const int64_t no = std::min<int64_t>((Cout + 31) / 32 * 32, C::NMAX);  // MMA N, multiple of 32
    pl->rows = static_cast<int>(no);
    pl->nK = static_cast<int>((Cin + eqlin::kChunkK16 - 1) / eqlin::kChunkK16);
    pl->n_oc = static_cast<int>((Cout + no - 1) / no);
    pl->BN = eqlin::tm::kM;
    pl->box_elems = C::X_BOX;
    pl->x_swizzle128 = C::X_SW128;
    const size_t wchunk = static_cast<size_t>(eqlin::pair_slots(G)) * no * eqlin::kRowBytes32;  // one (oc, c) chunk
    const size_t fixed = kSmemAlignSlack + kSmemCtlBytes +
                         static_cast<size_t>(eqlin::tm::kYStageBytes);
    if (pl->n_oc == 1) {
        const size_t img = wchunk * pl->nK;
        const size_t region = (img + 1023) / 1024 * 1024;
        if (max_smem > fixed + region) {
            const size_t stages = std::min<size_t>(kMaxStages, (max_smem - fixed - region) / C::XCHUNK_BYTES);
            if (stages >= 2) {
                pl->path = kPathTmResident;
                pl->stages = static_cast<int>(stages);
                pl->w_region_bytes = static_cast<uint32_t>(region);
                pl->w_img_bytes = static_cast<uint32_t>(img);
                pl->img_alloc_bytes = img;
                pl->smem_bytes = fixed + region + stages * C::XCHUNK_BYTES;
                return EQLIN_OK;
            }
        }
    }
    const size_t stage = C::XCHUNK_BYTES + wchunk;
    const size_t stages = max_smem > fixed ? std::min<size_t>(kMaxStages, (max_smem - fixed) / stage) : 0;
    if (stages < 1) return fail(EQLIN_ERR_UNSUPPORTED, "shape does not fit in shared memory");
    pl->path = kPathTmStreamed;
    pl->stages = static_cast<int>(stages);
    pl->w_region_bytes = 0;
    pl->w_img_bytes = 0;
    pl->img_alloc_bytes = wchunk * pl->nK * pl->n_oc;
    pl->smem_bytes = fixed + stages * stage;
    return EQLIN_OK;
}

// Kernel variant per group order, from B200 measurements: with tokens on M the MMA
// count per token no longer grows with the padding of a small Cout to 128 rows, which
// wins for G >= 8 (C16 C32: 358 -> 166 us, p8 C64: 30.9 -> 28.1 us); for G = 4 the
// double-buffered tokens-on-N kernel stays ahead (p4 C96: 70.1 vs 76.6 us).
bool default_tokens_on_m(int G) { return G >= 8; }

int plan_for(int64_t Cout, int64_t Cin, int64_t G, int io_dtype, size_t max_smem, Plan* pl) {
    pl->io = io_dtype;
    if (io_dtype == EQLIN_F32) {
        const size_t smem = static_cast<size_t>(eqlin::kF32Tokens) * G * Cin * sizeof(double);
        if (smem > max_smem) return fail(EQLIN_ERR_UNSUPPORTED, "Cin*G too large for the fp32 path");
        pl->path = kPathF32;
        pl->BN = eqlin::kF32Tokens;
        pl->smem_bytes = smem;
        return EQLIN_OK;
    }
    bool tm = default_tokens_on_m(static_cast<int>(G));
    bool tnr_ok = true;   // tokens on N: prefer the resident-input form when it applies
    bool tnr_forced = false;
    if (const char* e = std::getenv("EQLIN_KERNEL")) {
        if (std::strcmp(e, "tm") == 0) tm = true;
        if (std::strcmp(e, "tn") == 0) tm = false, tnr_ok = false;
        if (std::strcmp(e, "tnr") == 0) tm = false, tnr_forced = true;
    }
    if (!tm && tnr_ok) {
        int r = EQLIN_ERR_UNSUPPORTED;
        switch (G) {
            case 2: r = plan_tnr_g<2>(Cout, Cin, max_smem, tnr_forced, pl); break;
            case 4: r = plan_tnr_g<4>(Cout, Cin, max_smem, tnr_forced, pl); break;
            case 8: r = plan_tnr_g<8>(Cout, Cin, max_smem, tnr_forced, pl); break;
            case 16: r = plan_tnr_g<16>(Cout, Cin, max_smem, tnr_forced, pl); break;
            default: break;
        }
        if (r == EQLIN_OK) return EQLIN_OK;
    }
    if (tm) {
        switch (G) {
            case 2: return plan_tm_g<2>(Cout, Cin, max_smem, pl);
            case 4: return plan_tm_g<4>(Cout, Cin, max_smem, pl);
            case 8: return plan_tm_g<8>(Cout, Cin, max_smem, pl);
            case 16: return plan_tm_g<16>(Cout, Cin, max_smem, pl);
            default: return fail(EQLIN_ERR_UNSUPPORTED, "G must be 2, 4, 8 or 16");
        }
    }
    int nacc = 2;
    if (const char* e = std::getenv("EQLIN_ACC_BUFFERS")) {
        if (e[0] == '1') nacc = 1;
        if (e[0] == '2') nacc = 2;
    }
    switch (G) {
        case 2: return nacc == 1 ? plan_tn_g<2, 1>(Cout, Cin, max_smem, pl) : plan_tn_g<2, 2>(Cout, Cin, max_smem, pl);
        case 4: return nacc == 1 ? plan_tn_g<4, 1>(Cout, Cin, max_smem, pl) : plan_tn_g<4, 2>(Cout, Cin, max_smem, pl);
        case 8: return nacc == 1 ? plan_tn_g<8, 1>(Cout, Cin, max_smem, pl) : plan_tn_g<8, 2>(Cout, Cin, max_smem, pl);
        case 16: return nacc == 1 ? plan_tn_g<16, 1>(Cout, Cin, max_smem, pl) : plan_tn_g<16, 2>(Cout, Cin, max_smem, pl);
        default: return fail(EQLIN_ERR_UNSUPPORTED, "G must be 2, 4, 8 or 16");
    }
}

int check_shape_impl(int64_t Cout, int64_t Cin, int64_t G, int w_dtype, int io_dtype) {
    if (w_dtype != EQLIN_F32 && w_dtype != EQLIN_BF16 && w_dtype != EQLIN_F16)
        return fail(EQLIN_ERR_INVALID_ARG, "unknown w_dtype");
    if (io_dtype != EQLIN_F32 && io_dtype != EQLIN_BF16 && io_dtype != EQLIN_F16)
        return fail(EQLIN_ERR_INVALID_ARG, "unknown io_dtype");
    if (Cout <= 0 || Cin <= 0 || G <= 0) return fail(EQLIN_ERR_INVALID_ARG, "sizes must be positive");
    if (G != 2 && G != 4 && G != 8 && G != 16) return fail(EQLIN_ERR_UNSUPPORTED, "G must be 2, 4, 8 or 16");
    if (Cout > kMaxChannels || Cin > kMaxChannels) return fail(EQLIN_ERR_UNSUPPORTED, "channel count above 65536");
    if (io_dtype != EQLIN_F32 && ((Cin * G) % 8 != 0 || (Cout * G) % 8 != 0))
        return fail(EQLIN_ERR_UNSUPPORTED,
                     "16-bit I/O needs Cin*G and Cout*G to be multiples of 8 (16-byte rows)");
    return EQLIN_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// ------------------------------------------------------------- kernel tables
using TcLaunch = void (*)(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx,
                          const CUtensorMap& my, const TcParams& p);
using TmLaunch = void (*)(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx,
                          const CUtensorMap& my, const TmParams& p);

// The fused kernels are launched with programmatic stream serialization (PDL): a
// forward's CTAs may start while the previous kernel of the stream drains, and wait in
// griddepcontrol.wait before touching global memory.  Grids never exceed one CTA per
// SM, so a waiting dependent cannot starve its predecessor.  EQLIN_PDL=0 disables it.
bool use_pdl() {
    static const bool on = [] {
        const char* e = std::getenv("EQLIN_PDL");
        return !(e && e[0] == '0');
    }();
    return on;
}

template <class Kernel, class Params>
void launch_fused(Kernel k, unsigned grid, unsigned threads, size_t smem, cudaStream_t st, const CUtensorMap& mx,
                  const CUtensorMap& my, const Params& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = use_pdl() ? 1 : 0;
    cudaLaunchKernelEx(&cfg, k, mx, my, p);
}

template <int G, bool STREAM, int NACC, class T16>
void tc_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& my,
               const TcParams& p) {
    launch_fused(eqlin::eqlin_fwd_tc_kernel<G, STREAM, NACC, T16>, grid, eqlin::tc::kThreads, smem, st, mx, my, p);
}
template <int G, bool STREAM, class T16>
void tm_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& my,
               const TmParams& p) {
    launch_fused(eqlin::eqlin_fwd_tm_kernel<G, STREAM, T16>, grid, eqlin::tm::Cfg<G>::kThreads, smem, st, mx, my,
                 p);
}

struct TcEntry {
    TcLaunch launch = nullptr;
    void* kernel = nullptr;
};

template <int G, class T16>
void tcr_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& my,
                const TcParams& p) {
    launch_fused(eqlin::eqlin_fwd_tcr_kernel<G, T16>, grid, eqlin::tc::kThreads, smem, st, mx, my, p);
}
template <class T16>
TcEntry tcr_entry_t(int G) {
    switch (G) {
        case 2: return {&tcr_launch<2, T16>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tcr_kernel<2, T16>)};
        case 4: return {&tcr_launch<4, T16>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tcr_kernel<4, T16>)};
        case 8: return {&tcr_launch<8, T16>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tcr_kernel<8, T16>)};
        case 16: return {&tcr_launch<16, T16>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tcr_kernel<16, T16>)};
        default: return {};
    }
}
TcEntry tcr_entry_for(int G, int io) {
    return io == EQLIN_F16 ? tcr_entry_t<__half>(G) : tcr_entry_t<__nv_bfloat16>(G);
}
struct TmEntry {
    TmLaunch launch = nullptr;
    void* kernel = nullptr;
};

template <int G, bool STREAM, int NACC, class T16>
TcEntry tc_entry() {
    return {&tc_launch<G, STREAM, NACC, T16>,
            reinterpret_cast<void*>(&eqlin::eqlin_fwd_tc_kernel<G, STREAM, NACC, T16>)};
}
template <int G, class T16>
TcEntry tc_entry_g(bool stream, int nacc) {
    if (stream) return nacc == 1 ? tc_entry<G, true, 1, T16>() : tc_entry<G, true, 2, T16>();
    return nacc == 1 ? tc_entry<G, false, 1, T16>() : tc_entry<G, false, 2, T16>();
}
template <class T16>
TcEntry tc_entry_t(int G, bool stream, int nacc) {
    switch (G) {
        case 2: return tc_entry_g<2, T16>(stream, nacc);
        case 4: return tc_entry_g<4, T16>(stream, nacc);
        case 8: return tc_entry_g<8, T16>(stream, nacc);
        case 16: return tc_entry_g<16, T16>(stream, nacc);
        default: return {};
    }
}
TcEntry tc_entry_for(int G, bool stream, int nacc, int io) {
    return io == EQLIN_F16 ? tc_entry_t<__half>(G, stream, nacc) : tc_entry_t<__nv_bfloat16>(G, stream, nacc);
}

template <int G, bool STREAM, class T16>
TmEntry tm_entry() {
    return {&tm_launch<G, STREAM, T16>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tm_kernel<G, STREAM, T16>)};
}
template <class T16>
TmEntry tm_entry_t(int G, bool stream) {
    switch (G) {
        case 2: return stream ? tm_entry<2, true, T16>() : tm_entry<2, false, T16>();
        case 4: return stream ? tm_entry<4, true, T16>() : tm_entry<4, false, T16>();
        case 8: return stream ? tm_entry<8, true, T16>() : tm_entry<8, false, T16>();
        case 16: return stream ? tm_entry<16, true, T16>() : tm_entry<16, false, T16>();
        default: return {};
    }
}
TmEntry tm_entry_for(int G, bool stream, int io) {
    return io == EQLIN_F16 ? tm_entry_t<__half>(G, stream) : tm_entry_t<__nv_bfloat16>(G, stream);
}

void* f32_kernel_for(int G) {
    switch (G) {
        case 2: return reinterpret_cast<void*>(&eqlin::eqlin_fwd_f32_kernel<2>);
        case 4: return reinterpret_cast<void*>(&eqlin::eqlin_fwd_f32_kernel<4>);
        case 8: return reinterpret_cast<void*>(&eqlin::eqlin_fwd_f32_kernel<8>);
        case 16: return reinterpret_cast<void*>(&eqlin::eqlin_fwd_f32_kernel<16>);
        default: return nullptr;
    }
}

void* kernel_for(const Plan& pl, int G) {
    if (pl.path == kPathF32) return f32_kernel_for(G);
    if (pl.tm()) return tm_entry_for(G, pl.streamed(), pl.io).kernel;
    if (pl.tnr()) return tcr_entry_for(G, pl.io).kernel;
    return tc_entry_for(G, pl.streamed(), pl.nacc, pl.io).kernel;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// ------------------------------------------------------------------ launches
// Buffers of the frequency-domain weights (owned by a handle or carved from the
// allocation-free scratch array).
struct WeightBuffers {
    uint8_t* img = nullptr;       // bf16 tensor-core image (bf16 I/O)
    float* w_f32 = nullptr;       // [G][Cin][Cout]
    float* bias_f32 = nullptr;    // [Cout]
    double* w_f64 = nullptr;      // fp32-I/O path only
    double* bias_f64 = nullptr;   // fp32-I/O path only
    int* status = nullptr;
    bool has_bias = false;
    int act = eqlin::kActNone;   // epilogue activation of the forward (EQLIN_PREPARE_GELU)
    long long inject_stop = -1;  // failure-detection test hook (EQLIN_TEST_STOP_AFTER), -1 = off
};

// Cout x Cin is the operator's shape.  adjoint: the operator is the layer's input
// gradient (the layer's w is then [Cin, Cout, G] in these names, and bias is NULL).
int launch_prep(const Plan& pl, int w_dtype, const void* w, const void* bias, int64_t Cout, int64_t Cin,
                int64_t G, const WeightBuffers& b, cudaStream_t st, bool adjoint = false) {
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((Cout * Cin + threads - 1) / threads);
    const int iCout = static_cast<int>(Cout), iCin = static_cast<int>(Cin), iG = static_cast<int>(G);
    if (w_dtype == EQLIN_F32) {
        eqlin::eqlin_prep_freq_kernel<float><<<blocks, threads, 0, st>>>(
            static_cast<const float*>(w), static_cast<const float*>(bias), iCout, iCin, iG, b.w_f32, b.bias_f32,
            b.w_f64, b.bias_f64, adjoint);
    } else if (w_dtype == EQLIN_F16) {
        eqlin::eqlin_prep_freq_kernel<__half><<<blocks, threads, 0, st>>>(
            static_cast<const __half*>(w), static_cast<const __half*>(bias), iCout, iCin, iG, b.w_f32, b.bias_f32,
            b.w_f64, b.bias_f64, adjoint);
    } else {
        eqlin::eqlin_prep_freq_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(w), static_cast<const __nv_bfloat16*>(bias), iCout, iCin, iG,
            b.w_f32, b.bias_f32, b.w_f64, b.bias_f64, adjoint);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
    if (b.img) {
        const size_t n = pl.img_alloc_bytes / 2;
        const unsigned b2 = static_cast<unsigned>((n + threads - 1) / threads);
        const bool f16 = pl.io == EQLIN_F16;
        if (pl.tm() && f16) {
            eqlin::eqlin_prep_image_k16_kernel<__half><<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG, pl.nK,
                                                                                pl.rows, n, b.img);
        } else if (pl.tm()) {
            eqlin::eqlin_prep_image_k16_kernel<__nv_bfloat16><<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG,
                                                                                       pl.nK, pl.rows, n, b.img);
        } else if (f16) {
            eqlin::eqlin_prep_image_kernel<__half><<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG, pl.nK, pl.rows,
                                                                            n, b.img);
        } else {
            eqlin::eqlin_prep_image_kernel<__nv_bfloat16><<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG, pl.nK,
                                                                                   pl.rows, n, b.img);
        }
        e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "weight image launch");
    }
    return EQLIN_OK;
}

int launch_forward(const Plan& pl, int64_t Cout, int64_t Cin, int64_t G, int sm_count, const void* x, void* y,
                   int64_t N, const WeightBuffers& b, unsigned long long timeout_ns, cudaStream_t st) {
    const int iG = static_cast<int>(G);
    if (pl.path == kPathF32) {
        dim3 grid(static_cast<unsigned>((N + eqlin::kF32Tokens - 1) / eqlin::kF32Tokens),
                  static_cast<unsigned>((Cout + 31) / 32));
        const float* xf = static_cast<const float*>(x);
        float* yf = static_cast<float*>(y);
        const int iCin = static_cast<int>(Cin), iCout = static_cast<int>(Cout);
        switch (iG) {
            case 2: eqlin::eqlin_fwd_f32_kernel<2><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            case 4: eqlin::eqlin_fwd_f32_kernel<4><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            case 8: eqlin::eqlin_fwd_f32_kernel<8><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            default: eqlin::eqlin_fwd_f32_kernel<16><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
        }
    } else {
        auto encode = tensor_map_encoder();
        if (!encode) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        CUtensorMap map, ymap;
        cuuint32_t estr[2] = {1, 1};
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(Cin * G), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(Cin * G * 2)};
        cuuint32_t boxdim[2] = {static_cast<cuuint32_t>(pl.box_elems), static_cast<cuuint32_t>(pl.BN)};
        const CUtensorMapDataType dt16 =
            pl.io == EQLIN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
        CUresult r = encode(&map, dt16, 2, const_cast<void*>(x), dims, strides, boxdim,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            pl.x_swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
        cuuint64_t ydims[2] = {static_cast<cuuint64_t>(Cout * G), static_cast<cuuint64_t>(N)};
        cuuint64_t ystrides[1] = {static_cast<cuuint64_t>(Cout * G * 2)};
        cuuint32_t ybox[2];
        CUtensorMapSwizzle yswz;
        if (pl.tm()) {
            ybox[0] = eqlin::tm::kYCols;
            ybox[1] = eqlin::tm::kYRows;
            yswz = CU_TENSOR_MAP_SWIZZLE_64B;
        } else {
            ybox[0] = static_cast<cuuint32_t>(std::min<int64_t>(32 * G, eqlin::tc::kYBoxCols2));
            ybox[1] = static_cast<cuuint32_t>(pl.TG);
            yswz = CU_TENSOR_MAP_SWIZZLE_NONE;
        }
        r = encode(&ymap, dt16, 2, y, ydims, ystrides, ybox, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, yswz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for y");
        const long long n_tiles = (N + pl.BN - 1) / pl.BN;
        // the resident-input kernel's work item is a whole token tile (all output chunks)
        const int n_work = static_cast<int>(pl.tnr() ? n_tiles : n_tiles * pl.n_oc);
        const unsigned grid = static_cast<unsigned>(std::min<long long>(n_work, sm_count));
        if (pl.tm()) {
            TmParams p;
            p.w_img = b.img;
            p.bias = b.has_bias ? b.bias_f32 : nullptr;
            p.status = b.status;
            p.N = N;
            p.Cout = static_cast<int>(Cout);
            p.nK = pl.nK;
            p.NO = pl.rows;
            p.n_oc = pl.n_oc;
            p.n_work = n_work;
            p.stages = pl.stages;
            p.w_region_bytes = pl.w_region_bytes;
            p.w_img_bytes = pl.w_img_bytes;
            p.timeout_ns = timeout_ns;
            p.act = b.act;
            p.inject_stop = b.inject_stop;
            const TmEntry entry = tm_entry_for(iG, pl.streamed(), pl.io);
            if (!entry.launch) return fail(EQLIN_ERR_UNSUPPORTED, "G");
            entry.launch(grid, pl.smem_bytes, st, map, ymap, p);
        } else {
            TcParams p;
            p.w_img = b.img;
            p.bias = b.has_bias ? b.bias_f32 : nullptr;
            p.status = b.status;
            p.N = N;
            p.Cout = static_cast<int>(Cout);
            p.nK = pl.nK;
            p.rows = pl.rows;
            p.n_oc = pl.n_oc;
            p.n_work = n_work;
            p.stages = pl.stages;
            p.w_region_bytes = pl.w_region_bytes;
            p.ystage_bytes = pl.ystage_bytes;
            p.ybufs = pl.ybufs;
            p.y = static_cast<uint8_t*>(y);
            p.w_img_bytes = pl.w_img_bytes;
            p.timeout_ns = timeout_ns;
            p.act = b.act;
            p.inject_stop = b.inject_stop;
            const TcEntry entry = pl.tnr() ? tcr_entry_for(iG, pl.io) : tc_entry_for(iG, pl.streamed(), pl.nacc, pl.io);
            if (!entry.launch) return fail(EQLIN_ERR_UNSUPPORTED, "G");
            entry.launch(grid, pl.smem_bytes, st, map, ymap, p);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return EQLIN_OK;
}

// ------------------------------------------------------ weight gradient (dW)
// Tiling of the weight-gradient kernel: a unit is an (MO-row, NI-column) tile of the
// [Cout x Cin] gradient; the grid is units x token splits (see eqlin_bwd_dw.cuh).
struct DwPlan {
    int io = EQLIN_BF16;  // 16-bit element type of x and dy
    int MO = 0, NI = 0, n_ot = 0, n_it = 0, max_splits = 0;
    int MA = 0, NA = 0;   // 32-channel atoms of the MN-major spectra: ceil(MO / 32), ceil(NI / 32)
    int cpb_dy = 0, cpb_x = 0;
    int raw_stages = 0, spec_bufs = 0;
    int tok = 0;          // tokens per chunk (dw::Cfg<G>::kTok)
    uint32_t dy_bytes = 0, raw_bytes = 0, a_bytes = 0, b_bytes = 0, tmem_cols = 0;
    size_t smem_bytes = 0, slab_floats = 0;
    int units() const { return n_ot * n_it; }
};

uint32_t round_kb(size_t v) { return static_cast<uint32_t>((v + 1023) / 1024 * 1024); }
int round16(int64_t v) { return static_cast<int>((v + 15) / 16 * 16); }

// Channels per TMA box: the largest divisor d of C with d*G <= 256 elements, 16-byte
// box rows and d a multiple of `unit` (the channels of one transform unit); C is a
// multiple of 16, so d = 16 always qualifies.
int box_channels(int C, int G, int unit) {
    for (int d = C; d >= 1; --d)
        if (C % d == 0 && d % unit == 0 && d * G <= 256 && (d * G * 2) % 16 == 0) return d;
    return 0;
}

int dw_channels_per_unit(int G) { return G <= 4 ? 8 : (G == 8 ? 4 : 2); }

int max_dw_units(int G) {
    switch (G) {
        case 2: return eqlin::dw::Cfg<2>::kMaxPasses * eqlin::dw::Cfg<2>::kDftThreads;
        case 4: return eqlin::dw::Cfg<4>::kMaxPasses * eqlin::dw::Cfg<4>::kDftThreads;
        case 8: return eqlin::dw::Cfg<8>::kMaxPasses * eqlin::dw::Cfg<8>::kDftThreads;
        default: return eqlin::dw::Cfg<16>::kMaxPasses * eqlin::dw::Cfg<16>::kDftThreads;
    }
}

// Shared memory of the weight-gradient kernel: raw ring (RS stages of the 32-token dy and
// x tiles), SB spectra buffers (A: G dy planes of 4 K-groups x MA atoms of 512 B, plus
// the slack a 128-row MMA reads past the last plane; B: G x planes of 4 x NA atoms),
// the dbias slots [kTok tokens][MO] and the barriers.
// tokens per weight-gradient chunk, as the kernel instantiated for G uses them
int dw_tok(int G) {
    switch (G) {
        case 2: return eqlin::dw::Cfg<2>::kTok;
        case 4: return eqlin::dw::Cfg<4>::kTok;
        case 8: return eqlin::dw::Cfg<8>::kTok;
        default: return eqlin::dw::Cfg<16>::kTok;
    }
}

size_t dw_smem(int MO, int NI, int G, int RS, int SB, DwPlan* out) {
    const int MA = (MO + 31) / 32, NA = (NI + 31) / 32;
    const size_t raw = round_kb(static_cast<size_t>(dw_tok(G)) * (MO + NI) * G * 2);
    const int KG = dw_tok(G) / 8;
    // a 128-row MMA reads 4 atoms along M from each K group, MA of them written
    const size_t a = round_kb(static_cast<size_t>(G) * KG * MA * 512 + static_cast<size_t>(4 - MA) * 512);
    const size_t b = round_kb(static_cast<size_t>(G) * KG * NA * 512);
    const size_t total = kSmemAlignSlack + static_cast<size_t>(RS) * raw + static_cast<size_t>(SB) * (a + b) +
                         static_cast<size_t>(dw_tok(G)) * MO * 4 + 256;
    if (out) {
        out->MA = MA;
        out->NA = NA;
        out->dy_bytes = static_cast<uint32_t>(dw_tok(G)) * MO * G * 2;
        out->raw_bytes = static_cast<uint32_t>(raw);
        out->a_bytes = static_cast<uint32_t>(a);
        out->b_bytes = static_cast<uint32_t>(b);
        out->raw_stages = RS;
        out->spec_bufs = SB;
        out->tok = dw_tok(G);
        out->smem_bytes = total;
    }
    return total;
}

// Pick the tile with the fewest units that fits shared memory with the minimum
// pipeline (2 raw stages, 1 spectra buffer); fewer units = fewer re-reads of x and dy.
// Ties go to the larger MO (less MMA padding), then the larger NI.  Then the deepest
// raw ring that fits: with two spectra buffers (the transform of one chunk overlaps the
// MMAs of the previous one) when that still leaves >= 2 raw stages, else with one.  Tuning overrides: EQLIN_DW_TILE ("MO,NI"), EQLIN_DW_SPEC_BUFS,
// EQLIN_DW_RAW_STAGES.
int plan_dw(int64_t Cout, int64_t Cin, int G, size_t max_smem, int sm_count, DwPlan* pl) {
    const int mo_max = std::min(eqlin::kMmaM, round16(Cout));
    const int ni_cap = std::min(256, (512 / G) / 16 * 16);
    const int ni_max = std::min(ni_cap, round16(Cin));
    long long best_units = -1;
    int best_mo = 0, best_ni = 0;
    for (int mo = mo_max; mo >= 16; mo -= 16) {
        for (int ni = ni_max; ni >= 16; ni -= 16) {
            if (dw_smem(mo, ni, G, 2, 1, nullptr) > max_smem) continue;
            const long long units = ((Cout + mo - 1) / mo) * ((Cin + ni - 1) / ni);
            if (best_units < 0 || units < best_units) {
                best_units = units;
                best_mo = mo;
                best_ni = ni;
            }
        }
    }
    if (best_units < 0) return fail(EQLIN_ERR_UNSUPPORTED, "no weight-gradient tile fits shared memory");
    if (const char* e = std::getenv("EQLIN_DW_TILE")) {  // "MO,NI" tuning override
        int mo = 0, ni = 0;
        if (std::sscanf(e, "%d,%d", &mo, &ni) == 2 && mo >= 16 && mo <= mo_max && mo % 16 == 0 && ni >= 16 &&
            ni <= ni_max && ni % 16 == 0 && dw_smem(mo, ni, G, 2, 1, nullptr) <= max_smem) {
            best_mo = mo;
            best_ni = ni;
        }
    }
    auto max_rs = [&](int sb) {
        int rs = 0;
        while (rs < eqlin::dw::kMaxRawStages && dw_smem(best_mo, best_ni, G, rs + 1, sb, nullptr) <= max_smem) ++rs;
        return rs;
    };
    int sb = max_rs(2) >= 2 ? 2 : 1;
    const int sb_env = env_int("EQLIN_DW_SPEC_BUFS", 0);
    if (sb_env == 1 || (sb_env == 2 && max_rs(2) >= 2)) sb = sb_env;
    int rs = max_rs(sb);
    const int rs_env = env_int("EQLIN_DW_RAW_STAGES", 0);
    if (rs_env >= 2 && rs_env < rs) rs = rs_env;
    pl->MO = best_mo;
    pl->NI = best_ni;
    pl->n_ot = static_cast<int>((Cout + best_mo - 1) / best_mo);
    pl->n_it = static_cast<int>((Cin + best_ni - 1) / best_ni);
    pl->max_splits = std::max(1, sm_count / pl->units());
    // a transform unit (dw::Cfg<G>::kChanPerUnit channels) never straddles two boxes
    const int cpu = dw_channels_per_unit(G);
    pl->cpb_dy = box_channels(best_mo, G, cpu);
    pl->cpb_x = box_channels(best_ni, G, cpu);
    if (pl->cpb_dy == 0 || pl->cpb_x == 0) return fail(EQLIN_ERR_UNSUPPORTED, "no TMA box width for the tile");
    if (dw_tok(G) * (best_mo + best_ni) / cpu > max_dw_units(G))
        return fail(EQLIN_ERR_UNSUPPORTED, "weight-gradient tile has more transform units than threads can hold");
    dw_smem(best_mo, best_ni, G, rs, sb, pl);
    int cols = 32;
    while (cols < G * best_ni) cols *= 2;
    pl->tmem_cols = static_cast<uint32_t>(cols);
    pl->slab_floats = static_cast<size_t>(G) * best_ni * best_mo;
    return EQLIN_OK;
}

// Workspace of one weight-gradient call.  bf16 path: per CTA an fp32 slab ([G][NI][MO]
// partial planes, then [MO] bias sums).  fp32 path: a float64 [Cout][Cin][G] + [Cout]
// accumulator.
size_t dw_slab_region_bytes(const DwPlan& pl, int64_t N) {
    const long long n_chunks = (N + pl.tok - 1) / pl.tok;
    const long long splits = std::max<long long>(1, std::min<long long>(pl.max_splits, n_chunks));
    const size_t grid = static_cast<size_t>(pl.units()) * static_cast<size_t>(splits);
    const size_t bytes = grid * (pl.slab_floats + static_cast<size_t>(pl.MO)) * sizeof(float);
    return (bytes + 15) / 16 * 16;
}

size_t dw_workspace_bytes(const DwPlan& pl, bool f32_path, int64_t Cout, int64_t Cin, int64_t G, int64_t N) {
    if (f32_path) return static_cast<size_t>(Cout * Cin * G + Cout) * sizeof(double);
    return dw_slab_region_bytes(pl, N);
}

template <int G, class T16>
void dw_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mdy, const CUtensorMap& mx,
               const eqlin::DwParams& p) {
    launch_fused(eqlin::eqlin_dw_tc_kernel<G, T16>, grid, eqlin::dw::Cfg<G>::kThreads, smem, st, mdy, mx, p);
}

template <class T16>
void* dw_kernel_t(int G) {
    switch (G) {
        case 2: return reinterpret_cast<void*>(&eqlin::eqlin_dw_tc_kernel<2, T16>);
        case 4: return reinterpret_cast<void*>(&eqlin::eqlin_dw_tc_kernel<4, T16>);
        case 8: return reinterpret_cast<void*>(&eqlin::eqlin_dw_tc_kernel<8, T16>);
        case 16: return reinterpret_cast<void*>(&eqlin::eqlin_dw_tc_kernel<16, T16>);
        default: return nullptr;
    }
}
void* dw_kernel_for(int G, int io) { return io == EQLIN_F16 ? dw_kernel_t<__half>(G) : dw_kernel_t<__nv_bfloat16>(G); }

int encode_rows_map(CUtensorMap* map, const void* base, int64_t cols, int64_t rows, int box_cols, int box_rows,
                    int io) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint32_t estr[2] = {1, 1};
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    CUresult r = encode(map, io == EQLIN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    return EQLIN_OK;
}

int launch_dw(const DwPlan& pl, bool f32_path, int64_t Cout, int64_t Cin, int64_t G, const void* x, const void* dy,
              float* dw, float* dbias, int64_t N, void* ws, int* status, unsigned long long timeout_ns,
              cudaStream_t st) {
    const int iG = static_cast<int>(G), iCout = static_cast<int>(Cout), iCin = static_cast<int>(Cin);
    cudaError_t e;
    if (f32_path) {
        double* acc = static_cast<double*>(ws);
        const size_t n_w = static_cast<size_t>(Cout * Cin * G);
        if ((e = cudaMemsetAsync(acc, 0, (n_w + Cout) * sizeof(double), st)) != cudaSuccess)
            return cuda_fail(e, "weight-gradient accumulator clear");
        const long long pairs = Cout * Cin;
        const long long per = 512;
        const unsigned slices = static_cast<unsigned>(std::min<long long>((N + per - 1) / per, 65535));
        const long long tps = (N + slices - 1) / slices;
        dim3 grid(static_cast<unsigned>((pairs + 255) / 256), slices);
        const float* xf = static_cast<const float*>(x);
        const float* dyf = static_cast<const float*>(dy);
        switch (iG) {
            case 2: eqlin::eqlin_dw_f64_kernel<2><<<grid, 256, 0, st>>>(xf, dyf, acc, N, iCin, iCout, tps); break;
            case 4: eqlin::eqlin_dw_f64_kernel<4><<<grid, 256, 0, st>>>(xf, dyf, acc, N, iCin, iCout, tps); break;
            case 8: eqlin::eqlin_dw_f64_kernel<8><<<grid, 256, 0, st>>>(xf, dyf, acc, N, iCin, iCout, tps); break;
            default: eqlin::eqlin_dw_f64_kernel<16><<<grid, 256, 0, st>>>(xf, dyf, acc, N, iCin, iCout, tps); break;
        }
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "weight-gradient launch");
        const size_t n_conv = std::max(n_w, static_cast<size_t>(Cout));
        eqlin::eqlin_dw_f64_convert_kernel<<<static_cast<unsigned>((n_conv + 255) / 256), 256, 0, st>>>(
            acc, dw, dbias, n_w, iCout);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "weight-gradient convert launch");
        return EQLIN_OK;
    }
    CUtensorMap mdy, mx;
    int s = encode_rows_map(&mdy, dy, Cout * G, N, pl.cpb_dy * iG, dw_tok(G), pl.io);
    if (s != EQLIN_OK) return s;
    s = encode_rows_map(&mx, x, Cin * G, N, pl.cpb_x * iG, dw_tok(G), pl.io);
    if (s != EQLIN_OK) return s;
    eqlin::DwParams p;
    p.ws = static_cast<float*>(ws);
    p.status = status;
    p.N = N;
    p.MO = pl.MO;
    p.NI = pl.NI;
    p.n_it = pl.n_it;
    p.n_chunks = (N + dw_tok(G) - 1) / dw_tok(G);
    p.n_splits = static_cast<int>(std::max<long long>(1, std::min<long long>(pl.max_splits, p.n_chunks)));
    p.cpb_dy = pl.cpb_dy;
    p.cpb_x = pl.cpb_x;
    p.dy_bytes = pl.dy_bytes;
    p.raw_bytes = pl.raw_bytes;
    p.a_bytes = pl.a_bytes;
    p.b_bytes = pl.b_bytes;
    p.tmem_cols = pl.tmem_cols;
    p.raw_stages = pl.raw_stages;
    p.spec_bufs = pl.spec_bufs;
    p.slab_floats = pl.slab_floats;
    p.MA = pl.MA;
    p.NA = pl.NA;
    const unsigned grid = static_cast<unsigned>(pl.units() * p.n_splits);
    p.timeout_ns = timeout_ns;
    switch (iG) {
        case 2: pl.io == EQLIN_F16 ? dw_launch<2, __half>(grid, pl.smem_bytes, st, mdy, mx, p)
                                   : dw_launch<2, __nv_bfloat16>(grid, pl.smem_bytes, st, mdy, mx, p); break;
        case 4: pl.io == EQLIN_F16 ? dw_launch<4, __half>(grid, pl.smem_bytes, st, mdy, mx, p)
                                   : dw_launch<4, __nv_bfloat16>(grid, pl.smem_bytes, st, mdy, mx, p); break;
        case 8: pl.io == EQLIN_F16 ? dw_launch<8, __half>(grid, pl.smem_bytes, st, mdy, mx, p)
                                   : dw_launch<8, __nv_bfloat16>(grid, pl.smem_bytes, st, mdy, mx, p); break;
        default: pl.io == EQLIN_F16 ? dw_launch<16, __half>(grid, pl.smem_bytes, st, mdy, mx, p)
                                    : dw_launch<16, __nv_bfloat16>(grid, pl.smem_bytes, st, mdy, mx, p); break;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "weight-gradient launch");
    eqlin::DwFinalParams f;
    f.ws = p.ws;
    f.dw = dw;
    f.dbias = dbias;
    f.Cout = iCout;
    f.Cin = iCin;
    f.MO = pl.MO;
    f.NI = pl.NI;
    f.n_it = pl.n_it;
    f.n_splits = p.n_splits;
    f.slab_floats = pl.slab_floats;
    const unsigned fgrid = static_cast<unsigned>(pl.units() * (pl.NI + 1) * ((pl.MO + 31) / 32));
    switch (iG) {
        case 2: eqlin::eqlin_dw_finish_kernel<2><<<fgrid, 256, 0, st>>>(f); break;
        case 4: eqlin::eqlin_dw_finish_kernel<4><<<fgrid, 256, 0, st>>>(f); break;
        case 8: eqlin::eqlin_dw_finish_kernel<8><<<fgrid, 256, 0, st>>>(f); break;
        default: eqlin::eqlin_dw_finish_kernel<16><<<fgrid, 256, 0, st>>>(f); break;
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "weight-gradient reduction launch");
    return EQLIN_OK;
}

}  // namespace

namespace {
// Attributes that follow from the plans alone (shared by eqlin_get_attr and
// eqlin_query_plan); false when attr is not one of them.
bool plan_attr(const Plan& pl, const DwPlan& dwp, int64_t G, int64_t Cin, int64_t Cout, int io_dtype, int attr,
               int64_t* value) {
    const bool tn = pl.path == kPathResident || pl.path == kPathStreamed || pl.path == kPathTnResidentX;
    const bool has_dw = io_dtype != EQLIN_F32 && dwp.MO > 0;
    switch (attr) {
        case EQLIN_ATTR_G: *value = G; return true;
        case EQLIN_ATTR_CIN: *value = Cin; return true;
        case EQLIN_ATTR_COUT: *value = Cout; return true;
        case EQLIN_ATTR_IO_DTYPE: *value = io_dtype; return true;
        case EQLIN_ATTR_PATH: *value = pl.path; return true;
        case EQLIN_ATTR_TOKENS_PER_TILE: *value = pl.BN; return true;
        case EQLIN_ATTR_STAGES: *value = pl.stages; return true;
        case EQLIN_ATTR_SMEM_BYTES: *value = static_cast<int64_t>(pl.smem_bytes); return true;
        case EQLIN_ATTR_WEIGHT_BYTES:
            *value = pl.path == kPathF32 ? static_cast<int64_t>(G * Cin * Cout * 8)
                                         : static_cast<int64_t>(pl.img_alloc_bytes);
            return true;
        case EQLIN_ATTR_Y_STAGING: *value = tn ? pl.ybufs : -1; return true;
        case EQLIN_ATTR_DW_TILE_ROWS: *value = has_dw ? dwp.MO : -1; return true;
        case EQLIN_ATTR_DW_TILE_COLS: *value = has_dw ? dwp.NI : -1; return true;
        case EQLIN_ATTR_DW_RAW_STAGES: *value = has_dw ? dwp.raw_stages : -1; return true;
        case EQLIN_ATTR_DW_TOKENS: *value = has_dw ? dwp.tok : -1; return true;
        default: return false;
    }
}
}  // namespace

struct eqlin_handle {
    int device = 0;
    int sm_count = 0;
    int64_t Cout = 0, Cin = 0, G = 0;
    int w_dtype = 0, io_dtype = 0;
    Plan plan;
    WeightBuffers buf;   // device memory owned by the handle
    bool has_dx = false; // prepared with EQLIN_PREPARE_BACKWARD
    Plan plan_dx;        // input-gradient operator: [Cin x Cout], adjoint filters
    WeightBuffers buf_dx;  // its weights (status word shared with buf)
    DwPlan dwp;          // weight-gradient tiling (bf16 I/O)
    bool sync_check = false;
    unsigned long long timeout_ns = kDefaultTimeoutNs;
    // eqlin_forward_host: device staging for two chunks, two streams, created on first use
    std::mutex host_mutex;
    int64_t host_chunk = 0;                     // tokens per chunk (0: not set up)
    void* host_x[2] = {nullptr, nullptr};
    void* host_y[2] = {nullptr, nullptr};
    cudaStream_t host_st[2] = {nullptr, nullptr};
    cudaEvent_t host_ev_in = nullptr;
    cudaEvent_t host_ev_out[2] = {nullptr, nullptr};
};

namespace {

void release_host_staging(eqlin_handle* h) {
    for (int k = 0; k < 2; ++k) {
        if (h->host_x[k]) cudaFree(h->host_x[k]);
        if (h->host_y[k]) cudaFree(h->host_y[k]);
        if (h->host_st[k]) cudaStreamDestroy(h->host_st[k]);
        if (h->host_ev_out[k]) cudaEventDestroy(h->host_ev_out[k]);
        h->host_x[k] = h->host_y[k] = nullptr;
        h->host_st[k] = nullptr;
        h->host_ev_out[k] = nullptr;
    }
    if (h->host_ev_in) cudaEventDestroy(h->host_ev_in);
    h->host_ev_in = nullptr;
    h->host_chunk = 0;
}

void free_handle(eqlin_handle* h) {
    if (!h) return;
    if (h->buf.img) cudaFree(h->buf.img);
    if (h->buf.w_f32) cudaFree(h->buf.w_f32);
    if (h->buf.bias_f32) cudaFree(h->buf.bias_f32);
    if (h->buf.w_f64) cudaFree(h->buf.w_f64);
    if (h->buf.bias_f64) cudaFree(h->buf.bias_f64);
    if (h->buf.status) cudaFree(h->buf.status);
    if (h->buf_dx.img) cudaFree(h->buf_dx.img);
    if (h->buf_dx.w_f32) cudaFree(h->buf_dx.w_f32);
    if (h->buf_dx.bias_f32) cudaFree(h->buf_dx.bias_f32);
    if (h->buf_dx.w_f64) cudaFree(h->buf_dx.w_f64);
    if (h->buf_dx.bias_f64) cudaFree(h->buf_dx.bias_f64);
    release_host_staging(h);
    delete h;
}

size_t io_elem_bytes(int io) { return io == EQLIN_F32 ? 4 : 2; }

// Staging of eqlin_forward_host: chunks of about 16 MB of x plus y (a multiple of 64
// tokens), two of each, and two non-blocking streams.  Called with host_mutex held.
int setup_host_staging(eqlin_handle* h) {
    if (h->host_chunk > 0) return EQLIN_OK;
    const size_t e = io_elem_bytes(h->io_dtype);
    const size_t row_x = static_cast<size_t>(h->Cin * h->G) * e, row_y = static_cast<size_t>(h->Cout * h->G) * e;
    int64_t tokens = static_cast<int64_t>((size_t(16) << 20) / (row_x + row_y)) / 64 * 64;
    tokens = std::max<int64_t>(tokens, 64);
    cudaError_t err;
    for (int k = 0; k < 2; ++k) {
        if ((err = cudaMalloc(&h->host_x[k], tokens * row_x)) != cudaSuccess ||
            (err = cudaMalloc(&h->host_y[k], tokens * row_y)) != cudaSuccess) {
            cudaGetLastError();
            release_host_staging(h);   // nothing half set up survives a failure
            return fail(EQLIN_ERR_OOM, "staging allocation for the host-buffer forward");
        }
        if ((err = cudaStreamCreateWithFlags(&h->host_st[k], cudaStreamNonBlocking)) != cudaSuccess ||
            (err = cudaEventCreateWithFlags(&h->host_ev_out[k], cudaEventDisableTiming)) != cudaSuccess) {
            release_host_staging(h);
            return cuda_fail(err, "host-buffer forward streams");
        }
    }
    if ((err = cudaEventCreateWithFlags(&h->host_ev_in, cudaEventDisableTiming)) != cudaSuccess) {
        release_host_staging(h);
        return cuda_fail(err, "host-buffer forward streams");
    }
    h->host_chunk = tokens;
    return EQLIN_OK;
}

}  // namespace

extern "C" {

int eqlin_check_shape(int64_t Cout, int64_t Cin, int64_t G, int w_dtype, int io_dtype) {
    int s = check_shape_impl(Cout, Cin, G, w_dtype, io_dtype);
    if (s != EQLIN_OK) return s;
    Plan pl;
    return plan_for(Cout, Cin, G, io_dtype, kB200SmemOptin, &pl);
}

int eqlin_prepare_weights(const void* w, const void* bias, int64_t Cout, int64_t Cin, int64_t G, int w_dtype,
                          int io_dtype, void* stream, eqlin_handle** out) {
    return eqlin_prepare_weights_ex(w, bias, Cout, Cin, G, w_dtype, io_dtype, 0u, stream, out);
}

int eqlin_prepare_weights_ex(const void* w, const void* bias, int64_t Cout, int64_t Cin, int64_t G, int w_dtype,
                             int io_dtype, unsigned flags, void* stream, eqlin_handle** out) {
    if (!out) return fail(EQLIN_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
    if (flags & ~static_cast<unsigned>(EQLIN_PREPARE_BACKWARD | EQLIN_PREPARE_GELU))
        return fail(EQLIN_ERR_INVALID_ARG, "unknown flags");
    if (!w) return fail(EQLIN_ERR_INVALID_ARG, "w is NULL");
    int s = check_shape_impl(Cout, Cin, G, w_dtype, io_dtype);
    if (s != EQLIN_OK) return s;
    const size_t welt = w_dtype == EQLIN_F32 ? 4 : 2;
    if (!aligned(w, welt) || (bias && !aligned(bias, welt)))
        return fail(EQLIN_ERR_MISALIGNED, "w / bias not aligned to their element size");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    int major = 0, minor = 0, sms = 0, optin = 0;
    if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
        (e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return cuda_fail(e, "device query");
    if (major != 10 || minor != 0)
        return fail(EQLIN_ERR_UNSUPPORTED, "needs a compute capability 10.0 (sm_100a) device");

    Plan plan;
    s = plan_for(Cout, Cin, G, io_dtype, static_cast<size_t>(optin), &plan);
    if (s != EQLIN_OK) return s;

    eqlin_handle* h = new (std::nothrow) eqlin_handle();
    if (!h) return fail(EQLIN_ERR_OOM, "host allocation");
    h->device = dev;
    h->sm_count = sms;
    h->Cout = Cout;
    h->Cin = Cin;
    h->G = G;
    h->w_dtype = w_dtype;
    h->io_dtype = io_dtype;
    h->plan = plan;
    h->buf.has_bias = bias != nullptr;
    h->buf.act = (flags & EQLIN_PREPARE_GELU) ? eqlin::kActGelu : eqlin::kActNone;
    // Test hook for failure detection (read at prepare, never set outside tests): with
    // EQLIN_TEST_STOP_AFTER=k the fused kernels' producer stops after issuing k chunks per
    // CTA, so the consumers' bounded waits run out, the kernel records EQLIN_ERR_TIMEOUT
    // in the status word and exits cleanly.  No fault, trap or unbounded wait is involved.
    if (const char* e = std::getenv("EQLIN_TEST_STOP_AFTER")) {
        const long long k = std::atoll(e);
        if (k >= 0) h->buf.inject_stop = k;
    }
    const char* sc = std::getenv("EQLIN_SYNC_CHECK");
    h->sync_check = sc && sc[0] == '1';
    if (const char* t = std::getenv("EQLIN_WAIT_TIMEOUT_MS")) {
        const long long ms = std::atoll(t);
        if (ms > 0) h->timeout_ns = static_cast<unsigned long long>(ms) * 1000000ull;
    }

    const size_t wf_bytes = static_cast<size_t>(G) * Cin * Cout * sizeof(float);
    WeightBuffers& b = h->buf;
    if (cudaMalloc(&b.w_f32, wf_bytes) != cudaSuccess ||
        cudaMalloc(&b.bias_f32, static_cast<size_t>(Cout) * sizeof(float)) != cudaSuccess ||
        cudaMalloc(&b.status, 256) != cudaSuccess ||
        (plan.path == kPathF32 && (cudaMalloc(&b.w_f64, wf_bytes * 2) != cudaSuccess ||
                                   cudaMalloc(&b.bias_f64, static_cast<size_t>(Cout) * sizeof(double)) != cudaSuccess)) ||
        (plan.img_alloc_bytes && cudaMalloc(&b.img, plan.img_alloc_bytes) != cudaSuccess)) {
        cudaGetLastError();
        free_handle(h);
        return fail(EQLIN_ERR_OOM, "device allocation for the transformed weights");
    }
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if ((e = cudaMemsetAsync(b.status, 0, 256, st)) != cudaSuccess) {
        free_handle(h);
        return cuda_fail(e, "status init");
    }
    s = launch_prep(plan, w_dtype, w, bias, Cout, Cin, G, b, st);
    if (s == EQLIN_OK && (e = cudaStreamSynchronize(st)) != cudaSuccess) s = cuda_fail(e, "weight transform");
    if (s != EQLIN_OK) {
        free_handle(h);
        return s;
    }
    // The attribute is per kernel, not per handle: allow the device's opt-in maximum, so a
    // later handle of the same kernel with a smaller plan cannot lower it under this one.
    e = cudaFuncSetAttribute(kernel_for(plan, static_cast<int>(G)), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin);
    if (e != cudaSuccess) {
        free_handle(h);
        return cuda_fail(e, "cudaFuncSetAttribute");
    }
    if (flags & EQLIN_PREPARE_BACKWARD) {
        // input gradient: the same fused forward on the adjoint operator [Cin x Cout]
        s = plan_for(Cin, Cout, G, io_dtype, static_cast<size_t>(optin), &h->plan_dx);
        if (s != EQLIN_OK) {
            free_handle(h);
            return s;
        }
        WeightBuffers& d = h->buf_dx;
        const Plan& pd = h->plan_dx;
        d.status = b.status;
        d.has_bias = false;
        if (cudaMalloc(&d.w_f32, wf_bytes) != cudaSuccess ||
            cudaMalloc(&d.bias_f32, static_cast<size_t>(Cin) * sizeof(float)) != cudaSuccess ||
            (pd.path == kPathF32 && (cudaMalloc(&d.w_f64, wf_bytes * 2) != cudaSuccess ||
                                     cudaMalloc(&d.bias_f64, static_cast<size_t>(Cin) * sizeof(double)) != cudaSuccess)) ||
            (pd.img_alloc_bytes && cudaMalloc(&d.img, pd.img_alloc_bytes) != cudaSuccess)) {
            cudaGetLastError();
            free_handle(h);
            return fail(EQLIN_ERR_OOM, "device allocation for the input-gradient weights");
        }
        s = launch_prep(pd, w_dtype, w, nullptr, Cin, Cout, G, d, st, /*adjoint=*/true);
        if (s == EQLIN_OK && (e = cudaStreamSynchronize(st)) != cudaSuccess) s = cuda_fail(e, "input-gradient transform");
        if (s == EQLIN_OK &&
            (e = cudaFuncSetAttribute(kernel_for(pd, static_cast<int>(G)), cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      optin)) != cudaSuccess)
            s = cuda_fail(e, "cudaFuncSetAttribute");
        if (s != EQLIN_OK) {
            free_handle(h);
            return s;
        }
        h->has_dx = true;
    }
    if (io_dtype != EQLIN_F32) {
        // weight-gradient tiling (host only); a shape without one fails only in eqlin_backward_dw
        if (plan_dw(Cout, Cin, static_cast<int>(G), static_cast<size_t>(optin), sms, &h->dwp) == EQLIN_OK) {
            h->dwp.io = io_dtype;
            e = cudaFuncSetAttribute(dw_kernel_for(static_cast<int>(G), io_dtype),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, optin);
            if (e != cudaSuccess) {
                free_handle(h);
                return cuda_fail(e, "cudaFuncSetAttribute");
            }
        } else {
            h->dwp = DwPlan();
        }
        g_last_error.clear();
    }
    *out = h;
    return EQLIN_OK;
}

int eqlin_backward_dx(const eqlin_handle* h, const void* dy, void* dx, int64_t N, void* stream) {
    if (!h) return fail(EQLIN_ERR_INVALID_ARG, "handle is NULL");
    if (!h->has_dx) return fail(EQLIN_ERR_INVALID_ARG, "handle was prepared without EQLIN_PREPARE_BACKWARD");
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    if (N == 0) return EQLIN_OK;
    if (!dy || !dx) return fail(EQLIN_ERR_INVALID_ARG, "dy or dx is NULL");
    if (N >= (int64_t(1) << 31)) return fail(EQLIN_ERR_UNSUPPORTED, "N must be below 2^31");
    if (!aligned(dy, 16) || !aligned(dx, 16)) return fail(EQLIN_ERR_MISALIGNED, "dy and dx must be 16-byte aligned");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return fail(EQLIN_ERR_INVALID_ARG, "current device differs from the handle's device");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int s = launch_forward(h->plan_dx, h->Cin, h->Cout, h->G, h->sm_count, dy, dx, N, h->buf_dx, h->timeout_ns, st);
    if (s != EQLIN_OK) return s;
    if (h->sync_check) {
        int dst = 0;
        if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "backward_dx (EQLIN_SYNC_CHECK)");
        if ((e = cudaMemcpy(&dst, h->buf.status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
            return cuda_fail(e, "status read");
        if (dst != 0) return fail(dst, "device reported an error (status word)");
    }
    return EQLIN_OK;
}

int eqlin_backward_dw_workspace_size(const eqlin_handle* h, int64_t N, size_t* bytes) {
    if (!h || !bytes) return fail(EQLIN_ERR_INVALID_ARG, "NULL argument");
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    const bool f32_path = h->io_dtype == EQLIN_F32;
    if (!f32_path && h->dwp.MO == 0) return fail(EQLIN_ERR_UNSUPPORTED, "no weight-gradient tile for this shape");
    *bytes = N == 0 ? 0 : dw_workspace_bytes(h->dwp, f32_path, h->Cout, h->Cin, h->G, N);
    return EQLIN_OK;
}

int eqlin_backward_dw(const eqlin_handle* h, const void* x, const void* dy, float* dw, float* dbias, int64_t N,
                      void* workspace, size_t workspace_bytes, void* stream) {
    if (!h) return fail(EQLIN_ERR_INVALID_ARG, "handle is NULL");
    if (!dw) return fail(EQLIN_ERR_INVALID_ARG, "dw is NULL");
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    if (N >= (int64_t(1) << 31)) return fail(EQLIN_ERR_UNSUPPORTED, "N must be below 2^31");
    if (!aligned(dw, 4) || (dbias && !aligned(dbias, 4)))
        return fail(EQLIN_ERR_MISALIGNED, "dw and dbias must be 4-byte aligned");
    const bool f32_path = h->io_dtype == EQLIN_F32;
    if (!f32_path && h->dwp.MO == 0) return fail(EQLIN_ERR_UNSUPPORTED, "no weight-gradient tile for this shape");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return fail(EQLIN_ERR_INVALID_ARG, "current device differs from the handle's device");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t n_w = static_cast<size_t>(h->Cout * h->Cin * h->G);
    if (N == 0) {  // the gradient of an empty batch is zero
        if ((e = cudaMemsetAsync(dw, 0, n_w * sizeof(float), st)) != cudaSuccess) return cuda_fail(e, "dw clear");
        if (dbias && (e = cudaMemsetAsync(dbias, 0, static_cast<size_t>(h->Cout) * sizeof(float), st)) != cudaSuccess)
            return cuda_fail(e, "dbias clear");
        return EQLIN_OK;
    }
    if (!x || !dy) return fail(EQLIN_ERR_INVALID_ARG, "x or dy is NULL");
    if (!aligned(x, 16) || !aligned(dy, 16)) return fail(EQLIN_ERR_MISALIGNED, "x and dy must be 16-byte aligned");
    const size_t need = dw_workspace_bytes(h->dwp, f32_path, h->Cout, h->Cin, h->G, N);
    if (!workspace || workspace_bytes < need)
        return fail(EQLIN_ERR_INVALID_ARG, "workspace missing or smaller than eqlin_backward_dw_workspace_size (" +
                                               std::to_string(need) + " bytes)");
    if (!aligned(workspace, 16)) return fail(EQLIN_ERR_MISALIGNED, "workspace must be 16-byte aligned");
    int s = launch_dw(h->dwp, f32_path, h->Cout, h->Cin, h->G, x, dy, dw, dbias, N, workspace, h->buf.status,
                      h->timeout_ns, st);
    if (s != EQLIN_OK) return s;
    if (h->sync_check) {
        int dst = 0;
        if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "backward_dw (EQLIN_SYNC_CHECK)");
        if ((e = cudaMemcpy(&dst, h->buf.status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
            return cuda_fail(e, "status read");
        if (dst != 0) return fail(dst, "device reported an error (status word)");
    }
    return EQLIN_OK;
}

int eqlin_forward(const eqlin_handle* h, const void* x, void* y, int64_t N, void* stream) {
    if (!h) return fail(EQLIN_ERR_INVALID_ARG, "handle is NULL");
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    if (N == 0) return EQLIN_OK;
    if (!x || !y) return fail(EQLIN_ERR_INVALID_ARG, "x or y is NULL");
    if (N >= (int64_t(1) << 31)) return fail(EQLIN_ERR_UNSUPPORTED, "N must be below 2^31");
    if (!aligned(x, 16) || !aligned(y, 16)) return fail(EQLIN_ERR_MISALIGNED, "x and y must be 16-byte aligned");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return fail(EQLIN_ERR_INVALID_ARG, "current device differs from the handle's device");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int s = launch_forward(h->plan, h->Cout, h->Cin, h->G, h->sm_count, x, y, N, h->buf, h->timeout_ns, st);
    if (s != EQLIN_OK) return s;
    if (h->sync_check) {
        int dst = 0;
        e = cudaStreamSynchronize(st);
        if (e != cudaSuccess) return cuda_fail(e, "forward (EQLIN_SYNC_CHECK)");
        e = cudaMemcpy(&dst, h->buf.status, sizeof(int), cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return cuda_fail(e, "status read");
        if (dst != 0) return fail(dst, "device reported an error (status word)");
    }
    return EQLIN_OK;
}

int eqlin_forward_host(eqlin_handle* h, const void* x_host, void* y_host, int64_t N, void* stream) {
    if (!h) return fail(EQLIN_ERR_INVALID_ARG, "handle is NULL");
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    if (N == 0) return EQLIN_OK;
    if (!x_host || !y_host) return fail(EQLIN_ERR_INVALID_ARG, "x_host or y_host is NULL");
    if (N >= (int64_t(1) << 31)) return fail(EQLIN_ERR_UNSUPPORTED, "N must be below 2^31");
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev != h->device) return fail(EQLIN_ERR_INVALID_ARG, "current device differs from the handle's device");
    std::lock_guard<std::mutex> lock(h->host_mutex);
    int s = setup_host_staging(h);
    if (s != EQLIN_OK) return s;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const size_t el = io_elem_bytes(h->io_dtype);
    const size_t row_x = static_cast<size_t>(h->Cin * h->G) * el, row_y = static_cast<size_t>(h->Cout * h->G) * el;
    // both internal streams start after the work already queued on the caller's stream
    if ((e = cudaEventRecord(h->host_ev_in, st)) != cudaSuccess) return cuda_fail(e, "cudaEventRecord");
    for (int k = 0; k < 2; ++k)
        if ((e = cudaStreamWaitEvent(h->host_st[k], h->host_ev_in, 0)) != cudaSuccess)
            return cuda_fail(e, "cudaStreamWaitEvent");
    // chunk i on stream i % 2 with buffers i % 2: a stream's own order protects its
    // buffers, and the two streams overlap the copies in and out
    const auto* xb = static_cast<const uint8_t*>(x_host);
    auto* yb = static_cast<uint8_t*>(y_host);
    int64_t i = 0;
    for (int64_t n0 = 0; n0 < N; n0 += h->host_chunk, ++i) {
        const int k = static_cast<int>(i & 1);
        const int64_t n = std::min<int64_t>(h->host_chunk, N - n0);
        cudaStream_t sk = h->host_st[k];
        if ((e = cudaMemcpyAsync(h->host_x[k], xb + n0 * row_x, n * row_x, cudaMemcpyHostToDevice, sk)) !=
            cudaSuccess)
            return cuda_fail(e, "host-to-device copy");
        s = launch_forward(h->plan, h->Cout, h->Cin, h->G, h->sm_count, h->host_x[k], h->host_y[k], n, h->buf,
                           h->timeout_ns, sk);
        if (s != EQLIN_OK) return s;
        if ((e = cudaMemcpyAsync(yb + n0 * row_y, h->host_y[k], n * row_y, cudaMemcpyDeviceToHost, sk)) !=
            cudaSuccess)
            return cuda_fail(e, "device-to-host copy");
    }
    for (int k = 0; k < 2; ++k) {
        if ((e = cudaEventRecord(h->host_ev_out[k], h->host_st[k])) != cudaSuccess ||
            (e = cudaStreamWaitEvent(st, h->host_ev_out[k], 0)) != cudaSuccess)
            return cuda_fail(e, "stream join");
    }
    if (h->sync_check) {
        int dst = 0;
        if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "forward (EQLIN_SYNC_CHECK)");
        if ((e = cudaMemcpy(&dst, h->buf.status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
            return cuda_fail(e, "status read");
        if (dst != 0) return fail(dst, "device reported an error (status word)");
    }
    return EQLIN_OK;
}

int eqlin_destroy(eqlin_handle* h) {
    if (!h) return EQLIN_OK;
    free_handle(h);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "cudaFree");
    return EQLIN_OK;
}

int eqlin_device_status(eqlin_handle* h, int* status_out) {
    if (!h || !status_out) return fail(EQLIN_ERR_INVALID_ARG, "NULL argument");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int v = 0;
    if ((e = cudaMemcpy(&v, h->buf.status, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
        return cuda_fail(e, "status read");
    if ((e = cudaMemset(h->buf.status, 0, sizeof(int))) != cudaSuccess) return cuda_fail(e, "status clear");
    *status_out = v;
    return EQLIN_OK;
}

int eqlin_get_attr(const eqlin_handle* h, int attr, int64_t* value) {
    if (!h || !value) return fail(EQLIN_ERR_INVALID_ARG, "NULL argument");
    const Plan& pl = h->plan;
    if (plan_attr(pl, h->dwp, h->G, h->Cin, h->Cout, h->io_dtype, attr, value)) return EQLIN_OK;
    switch (attr) {
        case EQLIN_ATTR_G: *value = h->G; break;
        case EQLIN_ATTR_CIN: *value = h->Cin; break;
        case EQLIN_ATTR_COUT: *value = h->Cout; break;
        case EQLIN_ATTR_IO_DTYPE: *value = h->io_dtype; break;
        case EQLIN_ATTR_MAX_GRID: *value = pl.path == kPathF32 ? -1 : h->sm_count; break;
        case EQLIN_ATTR_ACTIVATION: *value = h->buf.act; break;
        default: return fail(EQLIN_ERR_INVALID_ARG, "unknown attribute");
    }
    return EQLIN_OK;
}

int eqlin_query_plan(int64_t Cout, int64_t Cin, int64_t G, int io_dtype, int attr, int64_t* value) {
    if (!value) return fail(EQLIN_ERR_INVALID_ARG, "NULL argument");
    int s = check_shape_impl(Cout, Cin, G, io_dtype, io_dtype);
    if (s != EQLIN_OK) return s;
    Plan pl;
    if ((s = plan_for(Cout, Cin, G, io_dtype, kB200SmemOptin, &pl)) != EQLIN_OK) return s;
    DwPlan dwp;
    if (io_dtype != EQLIN_F32 &&
        plan_dw(Cout, Cin, static_cast<int>(G), kB200SmemOptin, kB200SmCount, &dwp) != EQLIN_OK)
        dwp = DwPlan();
    if (attr == EQLIN_ATTR_MAX_GRID) {
        *value = pl.path == kPathF32 ? -1 : kB200SmCount;
        return EQLIN_OK;
    }
    if (plan_attr(pl, dwp, G, Cin, Cout, io_dtype, attr, value)) return EQLIN_OK;
    return fail(EQLIN_ERR_INVALID_ARG, "unknown attribute");
}

int eqlin_copy_freq_weights(const eqlin_handle* h, float* dst, int64_t count) {
    if (!h || !dst) return fail(EQLIN_ERR_INVALID_ARG, "NULL argument");
    const int64_t need = h->G * h->Cin * h->Cout;
    if (count < need) return fail(EQLIN_ERR_INVALID_ARG, "destination too small");
    cudaError_t e = cudaMemcpy(dst, h->buf.w_f32, static_cast<size_t>(need) * sizeof(float), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "copy of frequency-domain weights");
    return EQLIN_OK;
}

const char* eqlin_status_string(int status) {
    switch (status) {
        case EQLIN_OK: return "ok";
        case EQLIN_ERR_INVALID_ARG: return "invalid argument";
        case EQLIN_ERR_UNSUPPORTED: return "unsupported";
        case EQLIN_ERR_MISALIGNED: return "misaligned pointer";
        case EQLIN_ERR_CUDA: return "CUDA error";
        case EQLIN_ERR_OOM: return "out of memory";
        case EQLIN_ERR_TIMEOUT: return "device wait timed out";
        default: return "unknown status";
    }
}

const char* eqlin_last_error(void) { return g_last_error.c_str(); }

int eqlin_version(void) { return 100; }

}  // extern "C"

// ---------------------------------------------------------------------------------
// Allocation-free forward (eqlin_forward_noalloc).
//
// For callers that must not allocate device memory: a framework whose device memory
// is owned by its own pool (a stray cudaMalloc fragments it or is refused), or a host
// loop that cannot afford the implicit device-wide synchronisation and latency of
// cudaMalloc / cudaFree.  Such a caller passes only its inputs (x, w, bias) and its
// output (y); everything else the computation needs -- the device status word and the
// frequency-domain weights that eqlin_prepare_weights would keep in a handle -- lives
// in the fixed array below.  The array is part of the library image: every GPU that
// loads the library holds it until the process exits.
//
// In host code the array's name is only a host-side stand-in, never a device
// address, so its device address is looked up once per device (cudaGetSymbolAddress)
// and handed to the kernels as a pointer.
static __device__ __align__(256) unsigned char g_noalloc_scratch[EQLIN_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
constexpr int kNumPaths = 6;

struct NoAllocDevice {
    bool ready = false;
    uint8_t* scratch = nullptr;  // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    int optin = 0;
    bool cc_ok = false;
    uint8_t attr_done[kNumPaths][4][2][2] = {};  // [path][G index][nacc-1][fp16 I/O]: smem attribute set
};

std::mutex g_noalloc_mutex;
NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

int g_index(int64_t G) { return G == 2 ? 0 : G == 4 ? 1 : G == 8 ? 2 : 3; }

// First call on a device, with that device current: resolve the scratch array's
// device address and read the device limits.  Later calls reuse them.
int noalloc_setup(int dev, NoAllocDevice** out) {
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(EQLIN_ERR_UNSUPPORTED, "device index above 63");
    NoAllocDevice& d = g_noalloc_dev[dev];
    if (!d.ready) {
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
        int major = 0, minor = 0;
        if ((e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
            (e = cudaDeviceGetAttribute(&d.optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return cuda_fail(e, "device query");
        d.cc_ok = major == 10 && minor == 0;
        d.scratch = static_cast<uint8_t*>(ptr);
        d.ready = true;
    }
    if (!d.cc_ok) return fail(EQLIN_ERR_UNSUPPORTED, "needs a compute capability 10.0 (sm_100a) device");
    *out = &d;
    return EQLIN_OK;
}

}  // namespace

extern "C" int eqlin_forward_noalloc(const void* x, const void* w, const void* bias, void* y, int64_t N,
                                     int64_t Cout, int64_t Cin, int64_t G, int dtype, void* stream) {
    int s = check_shape_impl(Cout, Cin, G, dtype, dtype);
    if (s != EQLIN_OK) return s;
    if (N < 0) return fail(EQLIN_ERR_INVALID_ARG, "N < 0");
    if (!w) return fail(EQLIN_ERR_INVALID_ARG, "w is NULL");
    if (N == 0) return EQLIN_OK;
    if (!x || !y) return fail(EQLIN_ERR_INVALID_ARG, "x or y is NULL");
    if (N >= (int64_t(1) << 31)) return fail(EQLIN_ERR_UNSUPPORTED, "N must be below 2^31");
    const size_t elt = dtype == EQLIN_F32 ? 4 : 2;
    if (!aligned(x, 16) || !aligned(y, 16)) return fail(EQLIN_ERR_MISALIGNED, "x and y must be 16-byte aligned");
    if (!aligned(w, elt) || (bias && !aligned(bias, elt)))
        return fail(EQLIN_ERR_MISALIGNED, "w / bias not aligned to their element size");

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    NoAllocDevice* d = nullptr;
    Plan plan;
    {
        std::lock_guard<std::mutex> lock(g_noalloc_mutex);
        s = noalloc_setup(dev, &d);
        if (s != EQLIN_OK) return s;
        s = plan_for(Cout, Cin, G, dtype, static_cast<size_t>(d->optin), &plan);
        if (s != EQLIN_OK) return s;
        // kernel shared-memory attribute (the device's opt-in maximum), once per kernel and device
        uint8_t& done = d->attr_done[plan.path][g_index(G)][plan.nacc == 1 ? 0 : 1][dtype == EQLIN_F16 ? 1 : 0];
        if (!done) {
            e = cudaFuncSetAttribute(kernel_for(plan, static_cast<int>(G)),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, d->optin);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");
            done = 1;
        }
    }

    // scratch layout: status word | fp32 bias | fp32 planes | (bf16 image | fp64 planes + bias)
    const size_t planes = static_cast<size_t>(G) * Cin * Cout;
    size_t off = 0;
    const size_t off_status = off;
    off += 256;
    const size_t off_bias = off;
    off = align256(off + static_cast<size_t>(Cout) * sizeof(float));
    const size_t off_wf = off;
    off = align256(off + planes * sizeof(float));
    size_t off_img = 0, off_wd = 0, off_bd = 0;
    if (plan.path == kPathF32) {
        off_wd = off;
        off = align256(off + planes * sizeof(double));
        off_bd = off;
        off = align256(off + static_cast<size_t>(Cout) * sizeof(double));
    } else {
        off_img = off;
        off = align256(off + plan.img_alloc_bytes);
    }
    if (off > EQLIN_NOALLOC_SCRATCH_BYTES)
        return fail(EQLIN_ERR_UNSUPPORTED, "shape needs " + std::to_string(off) +
                                               " bytes of scratch; eqlin_forward_noalloc is limited to " +
                                               std::to_string(EQLIN_NOALLOC_SCRATCH_BYTES));
    uint8_t* sc = d->scratch;
    WeightBuffers b;
    b.status = reinterpret_cast<int*>(sc + off_status);
    b.bias_f32 = reinterpret_cast<float*>(sc + off_bias);
    b.w_f32 = reinterpret_cast<float*>(sc + off_wf);
    b.w_f64 = plan.path == kPathF32 ? reinterpret_cast<double*>(sc + off_wd) : nullptr;
    b.bias_f64 = plan.path == kPathF32 ? reinterpret_cast<double*>(sc + off_bd) : nullptr;
    b.img = plan.path == kPathF32 ? nullptr : sc + off_img;
    b.has_bias = bias != nullptr;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    // the status word keeps the previous call's value: clear it
    if ((e = cudaMemsetAsync(b.status, 0, sizeof(int), st)) != cudaSuccess) return cuda_fail(e, "status clear");
    // weight transform into the scratch, then the forward (same kernels as the handle API)
    s = launch_prep(plan, dtype, w, bias, Cout, Cin, G, b, st);
    if (s != EQLIN_OK) return s;
    return launch_forward(plan, Cout, Cin, G, d->sm_count, x, y, N, b, kDefaultTimeoutNs, st);
}
