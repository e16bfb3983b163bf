// eqlin_host_plan.h -- host-side planning of the kernels (included once, by eqlin_api.cu,
// after the CUDA and kernel headers), with the error helpers:
// shared-memory budget, ring depth, kernel form and y store mode of the forward, and the
// tiling of the weight gradient.  Host only; eqlin_query_plan exposes the result without
// a GPU.
#pragma once

namespace {

constexpr size_t kB200SmemOptin = 232448;   // 227 KB opt-in shared memory per CTA on sm_100
constexpr int kB200SmCount = 148;           // SMs of a B200 (host-only planning queries)
constexpr size_t kSmemAlignSlack = 1024;    // the kernels round their smem base up to 1 KB
constexpr size_t kSmemCtlBytes = 512;       // mbarriers + control block
constexpr int kMaxStages = 12;
constexpr int64_t kMaxChannels = 1 << 16;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait
// L2 prefetch distance of the fused kernels (work items).  Off: on B200 every workload was
// slower with it (200 back-to-back launches, distance 2 / 0: p4 C96 63.1 / 62.1 us, p8 C64
// 24.2 / 22.8, p4 192->768 189.6 / 181.5, C16 C32 153.4 / 145.6).
constexpr int kDefaultPrefetch = 0;
constexpr bool kDefaultL2Hint = true;   // L2 eviction priorities on the fused kernels' copies

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
    int TG = 0;          // y TMA store box rows (tokens-on-N): the epilogue group's tokens
    int ybufs = 0;       // y staging buffers per epilogue warp (tokens-on-N)
    int yq = 4;          // TMEM lane quarters with output rows, each given y staging (tokens-on-N)
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
    pl->box_elems = S::BOX_ELEMS;
    // Only the TMEM lane quarters that hold output rows get y staging (Cout = 96 leaves the
    // fourth one empty), and the freed space deepens the input ring.
    pl->yq = pl->n_oc == 1 ? static_cast<int>((Cout + 31) / 32) : 4;
    pl->TG = S::TG;
    // y staging: per active epilogue warp, ybufs buffers of TG rows x 32*G 16-bit columns;
    // double-buffered when at least 4 ring stages still fit (B200, p4 C96: 3 stages 72.5 us,
    // 4 stages 60.9 us, 5 stages 60.1 us)
    const size_t ybuf = static_cast<size_t>(pl->TG) * 32 * G * 2;
    auto fixed_for = [&](int nb) {
        return kSmemAlignSlack + kSmemCtlBytes + static_cast<size_t>(2 * pl->yq) * nb * ybuf;
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
        pl->yq = 4;
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
    const size_t wchunk = static_cast<size_t>(eqlin::tm_weight_slots(G)) * no * eqlin::kRowBytes32;  // one (oc, c) chunk
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

// `act`: the forward's epilogue activation.  With GELU the epilogue is ALU-bound, and the
// resident-input form (x transformed once per tile, not once per output chunk) wins from 2
// input chunks on and for G = 8 too (B200, 20 GELU layers back to back: p4 96 -> 384 309.2
// vs 324.6 us streamed, 64 -> 256 206.6 vs 210.5, 96 -> 256 211.8 vs 219.5; G = 8 64 -> 256
// 59.0 vs 67.8 us tokens on M at N = 25088, 198.2 vs 231.2 at 100352), while without an
// activation the rules below stand (96 -> 384: 191.4 vs 180.2 us).
int plan_for(int64_t Cout, int64_t Cin, int64_t G, int io_dtype, size_t max_smem, Plan* pl,
             int act = eqlin::kActNone) {
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
    const bool gelu_tnr = act == eqlin::kActGelu && G <= 8 && Cout > eqlin::kMmaM && Cin > eqlin::kChunkK;
    if (const char* e = std::getenv("EQLIN_KERNEL")) {
        if (std::strcmp(e, "tm") == 0) tm = true;
        if (std::strcmp(e, "tn") == 0) tm = false, tnr_ok = false;
        if (std::strcmp(e, "tnr") == 0) tm = false, tnr_forced = true;
    } else if (gelu_tnr) {
        int r = EQLIN_ERR_UNSUPPORTED;
        switch (G) {
            case 2: r = plan_tnr_g<2>(Cout, Cin, max_smem, true, pl); break;
            case 4: r = plan_tnr_g<4>(Cout, Cin, max_smem, true, pl); break;
            case 8: r = plan_tnr_g<8>(Cout, Cin, max_smem, true, pl); break;
            default: break;
        }
        if (r == EQLIN_OK) return EQLIN_OK;
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
// pipeline (2 raw stages, 1 spectra buffer) and whose transform units the threads can
// hold; fewer units = fewer re-reads of x and dy.  Ties go to the least padded area (192
// input channels as 2 x 96, not 128 + 64: B200, weight gradient of the 192 -> 768 layer
// 341 us against 386 us), then to the larger MO (less MMA padding), then the larger NI.  Then the deepest
// raw ring that fits: with two spectra buffers (the transform of one chunk overlaps the
// MMAs of the previous one) when that still leaves >= 2 raw stages, else with one.
// Tuning overrides: EQLIN_DW_TILE ("MO,NI"), EQLIN_DW_SPEC_BUFS, EQLIN_DW_RAW_STAGES.
int plan_dw(int64_t Cout, int64_t Cin, int G, size_t max_smem, int sm_count, DwPlan* pl) {
    const int mo_max = std::min(eqlin::kMmaM, round16(Cout));
    const int ni_cap = std::min(256, (512 / G) / 16 * 16);
    const int ni_max = std::min(ni_cap, round16(Cin));
    long long best_units = -1, best_area = 0;
    int best_mo = 0, best_ni = 0;
    const int cpu = dw_channels_per_unit(G);
    for (int mo = mo_max; mo >= 16; mo -= 16) {
        for (int ni = ni_max; ni >= 16; ni -= 16) {
            if (dw_tok(G) * (mo + ni) / cpu > max_dw_units(G)) continue;
            if (dw_smem(mo, ni, G, 2, 1, nullptr) > max_smem) continue;
            const long long n_ot = (Cout + mo - 1) / mo, n_it = (Cin + ni - 1) / ni;
            const long long units = n_ot * n_it, area = n_ot * mo * n_it * ni;
            if (best_units < 0 || units < best_units || (units == best_units && area < best_area)) {
                best_units = units;
                best_area = area;
                best_mo = mo;
                best_ni = ni;
            }
        }
    }
    if (best_units < 0) return fail(EQLIN_ERR_UNSUPPORTED, "no weight-gradient tile fits shared memory");
    if (const char* e = std::getenv("EQLIN_DW_TILE")) {  // "MO,NI" tuning override
        int mo = 0, ni = 0;
        if (std::sscanf(e, "%d,%d", &mo, &ni) == 2 && mo >= 16 && mo <= mo_max && mo % 16 == 0 && ni >= 16 &&
            ni <= ni_max && ni % 16 == 0 && dw_smem(mo, ni, G, 2, 1, nullptr) <= max_smem &&
            dw_tok(G) * (mo + ni) / cpu <= max_dw_units(G)) {
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
    // raw boxes of 128-byte rows (64 at G = 2), swizzled (dw::Cfg<G>::kRowBytes): MO and NI,
    // multiples of 16, are multiples of the box's channels
    pl->cpb_dy = pl->cpb_x = (G == 2 ? 64 : 128) / (2 * G);
    if (best_mo % pl->cpb_dy != 0 || best_ni % pl->cpb_x != 0 || pl->cpb_dy % cpu != 0)
        return fail(EQLIN_ERR_UNSUPPORTED, "no TMA box width for the tile");
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
