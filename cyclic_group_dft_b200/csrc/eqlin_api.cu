// eqlin_api.cu -- host side of the C ABI declared in include/eqlin.h: argument
// validation, kernel planning (shared-memory budget, ring depth, kernel variant),
// ownership of the frequency-domain weights, TMA descriptor encoding and launches.
#include "eqlin.h"

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <string>

#include "eqlin_fwd_tc.cuh"
#include "eqlin_fwd_tm.cuh"
#include "eqlin_layout.h"
#include "eqlin_prep.cuh"

using eqlin::TcParams;
using eqlin::TmParams;

namespace {

constexpr size_t kB200SmemOptin = 232448;   // 227 KB opt-in shared memory per CTA on sm_100
constexpr size_t kSmemAlignSlack = 1024;    // the kernels round their smem base up to 1 KB
constexpr size_t kSmemCtlBytes = 512;       // mbarriers + control block
constexpr int kMaxStages = 12;
constexpr int64_t kMaxChannels = 1 << 16;
constexpr unsigned long long kDefaultTimeoutNs = 2000000000ull;  // 2 s per bounded wait

// Kernel variants (EQLIN_ATTR_PATH):
//   0/1  tcgen05, tokens on the MMA N dimension, weights resident / streamed
//   2    fp32 I/O, float64 CUDA-core kernel
//   3/4  tcgen05, tokens on the MMA M dimension, weights resident / streamed
enum Path { kPathResident = 0, kPathStreamed = 1, kPathF32 = 2, kPathTmResident = 3, kPathTmStreamed = 4 };

thread_local std::string g_last_error;

int fail(int code, const std::string& msg) {
    g_last_error = msg;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(EQLIN_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

struct Plan {
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
    uint32_t w_region_bytes = 0, w_img_bytes = 0, ystage_bytes = 0;
    size_t smem_bytes = 0;
    size_t img_alloc_bytes = 0;
    bool tm() const { return path == kPathTmResident || path == kPathTmStreamed; }
    bool streamed() const { return path == kPathStreamed || path == kPathTmStreamed; }
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

template <int G, int NACC>
int plan_tn_g(int64_t Cout, int64_t Cin, size_t max_smem, Plan* pl) {
    const int max_stages = std::min(kMaxStages, env_int("EQLIN_MAX_STAGES", kMaxStages));
    const int ybufs_env = env_int("EQLIN_YBUFS", 0);
    using S = eqlin::tc::Shape<G, NACC>;
    pl->nacc = NACC;
    pl->nK = static_cast<int>((Cin + eqlin::kChunkK - 1) / eqlin::kChunkK);
    pl->n_oc = static_cast<int>((Cout + eqlin::kMmaM - 1) / eqlin::kMmaM);
    pl->BN = S::BN;
    pl->TG = S::TG;
    pl->box_elems = S::BOX_ELEMS;
    // y staging: per epilogue warp, ybufs buffers of TG rows x 32*G bf16 columns (4 KB);
    // double-buffered when at least 5 ring stages still fit
    const size_t ybuf = static_cast<size_t>(S::TG) * 32 * G * 2;
    auto fixed_for = [&](int nb) {
        return kSmemAlignSlack + kSmemCtlBytes + static_cast<size_t>(eqlin::tc::kEpiWarps) * nb * ybuf;
    };
    pl->ybufs = 2;
    for (int nb = 2; nb >= 1; --nb) {
        if (ybufs_env && nb != ybufs_env) continue;
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
                    std::min<size_t>(max_stages, (max_smem - fixed - region) / S::XCHUNK_BYTES);
                if (stages >= static_cast<size_t>(nb == 2 && !ybufs_env ? 5 : 2)) {
                    pl->path = kPathResident;
                    pl->rows = rows;
                    pl->stages = static_cast<int>(stages);
                    pl->w_region_bytes = static_cast<uint32_t>(region);
                    pl->w_img_bytes = static_cast<uint32_t>(img);
                    pl->img_alloc_bytes = img;
                    pl->smem_bytes = fixed + region + stages * S::XCHUNK_BYTES;
                    return EQLIN_OK;
                }
            }
        }
        // weights streamed chunk by chunk next to each x chunk
        if (pl->n_oc > 1 || nb == 1) {
            const size_t stage = static_cast<size_t>(S::XCHUNK_BYTES) + S::WSTAGE_BYTES;
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

template <int G>
int plan_tm_g(int64_t Cout, int64_t Cin, size_t max_smem, Plan* pl) {
    using C = eqlin::tm::Cfg<G>;
    const int kMaxStages = std::min(::kMaxStages, env_int("EQLIN_MAX_STAGES", ::kMaxStages));
    const int64_t no = std::min<int64_t>((Cout + 31) / 32 * 32, C::NMAX);  // MMA N, multiple of 32
    pl->rows = static_cast<int>(no);
    pl->nK = static_cast<int>((Cin + eqlin::kChunkK16 - 1) / eqlin::kChunkK16);
    pl->n_oc = static_cast<int>((Cout + no - 1) / no);
    pl->BN = eqlin::tm::kM;
    pl->box_elems = C::XROW_ELEMS;
    const size_t wchunk = static_cast<size_t>(G) * no * eqlin::kRowBytes32;   // one (oc, c) weight chunk
    const size_t fixed = kSmemAlignSlack + kSmemCtlBytes +
                         static_cast<size_t>(eqlin::tm::kYBufs) * eqlin::tm::kYBufBytes;
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
    if (io_dtype == EQLIN_F32) {
        const size_t smem = static_cast<size_t>(eqlin::kF32Tokens) * G * Cin * sizeof(double);
        if (smem > max_smem) return fail(EQLIN_ERR_UNSUPPORTED, "Cin*G too large for the fp32 path");
        pl->path = kPathF32;
        pl->BN = eqlin::kF32Tokens;
        pl->smem_bytes = smem;
        return EQLIN_OK;
    }
    bool tm = default_tokens_on_m(static_cast<int>(G));
    if (const char* e = std::getenv("EQLIN_KERNEL")) {
        if (std::strcmp(e, "tm") == 0) tm = true;
        if (std::strcmp(e, "tn") == 0) tm = false;
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
    if (w_dtype != EQLIN_F32 && w_dtype != EQLIN_BF16) return fail(EQLIN_ERR_INVALID_ARG, "unknown w_dtype");
    if (io_dtype != EQLIN_F32 && io_dtype != EQLIN_BF16) return fail(EQLIN_ERR_INVALID_ARG, "unknown io_dtype");
    if (Cout <= 0 || Cin <= 0 || G <= 0) return fail(EQLIN_ERR_INVALID_ARG, "sizes must be positive");
    if (G != 2 && G != 4 && G != 8 && G != 16) return fail(EQLIN_ERR_UNSUPPORTED, "G must be 2, 4, 8 or 16");
    if (Cout > kMaxChannels || Cin > kMaxChannels) return fail(EQLIN_ERR_UNSUPPORTED, "channel count above 65536");
    if (io_dtype == EQLIN_BF16 && ((Cin * G) % 8 != 0 || (Cout * G) % 8 != 0))
        return fail(EQLIN_ERR_UNSUPPORTED, "bf16 I/O needs Cin*G and Cout*G to be multiples of 8 (16-byte rows)");
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

template <int G, bool STREAM, int NACC>
void tc_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& my,
               const TcParams& p) {
    launch_fused(eqlin::eqlin_fwd_tc_kernel<G, STREAM, NACC>, grid, eqlin::tc::kThreads, smem, st, mx, my, p);
}
template <int G, bool STREAM>
void tm_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const CUtensorMap& my,
               const TmParams& p) {
    launch_fused(eqlin::eqlin_fwd_tm_kernel<G, STREAM>, grid, eqlin::tm::Cfg<G>::kThreads, smem, st, mx, my, p);
}

struct TcEntry {
    TcLaunch launch = nullptr;
    void* kernel = nullptr;
};
struct TmEntry {
    TmLaunch launch = nullptr;
    void* kernel = nullptr;
};

template <int G, bool STREAM, int NACC>
TcEntry tc_entry() {
    return {&tc_launch<G, STREAM, NACC>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tc_kernel<G, STREAM, NACC>)};
}
template <int G>
TcEntry tc_entry_g(bool stream, int nacc) {
    if (stream) return nacc == 1 ? tc_entry<G, true, 1>() : tc_entry<G, true, 2>();
    return nacc == 1 ? tc_entry<G, false, 1>() : tc_entry<G, false, 2>();
}
TcEntry tc_entry_for(int G, bool stream, int nacc) {
    switch (G) {
        case 2: return tc_entry_g<2>(stream, nacc);
        case 4: return tc_entry_g<4>(stream, nacc);
        case 8: return tc_entry_g<8>(stream, nacc);
        case 16: return tc_entry_g<16>(stream, nacc);
        default: return {};
    }
}

template <int G, bool STREAM>
TmEntry tm_entry() {
    return {&tm_launch<G, STREAM>, reinterpret_cast<void*>(&eqlin::eqlin_fwd_tm_kernel<G, STREAM>)};
}
TmEntry tm_entry_for(int G, bool stream) {
    switch (G) {
        case 2: return stream ? tm_entry<2, true>() : tm_entry<2, false>();
        case 4: return stream ? tm_entry<4, true>() : tm_entry<4, false>();
        case 8: return stream ? tm_entry<8, true>() : tm_entry<8, false>();
        case 16: return stream ? tm_entry<16, true>() : tm_entry<16, false>();
        default: return {};
    }
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
    if (pl.tm()) return tm_entry_for(G, pl.streamed()).kernel;
    return tc_entry_for(G, pl.streamed(), pl.nacc).kernel;
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
};

int launch_prep(const Plan& pl, int w_dtype, const void* w, const void* bias, int64_t Cout, int64_t Cin,
                int64_t G, const WeightBuffers& b, cudaStream_t st) {
    const int threads = 256;
    const unsigned blocks = static_cast<unsigned>((Cout * Cin + threads - 1) / threads);
    const int iCout = static_cast<int>(Cout), iCin = static_cast<int>(Cin), iG = static_cast<int>(G);
    if (w_dtype == EQLIN_F32) {
        eqlin::eqlin_prep_freq_kernel<float><<<blocks, threads, 0, st>>>(
            static_cast<const float*>(w), static_cast<const float*>(bias), iCout, iCin, iG, b.w_f32, b.bias_f32,
            b.w_f64, b.bias_f64);
    } else {
        eqlin::eqlin_prep_freq_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
            static_cast<const __nv_bfloat16*>(w), static_cast<const __nv_bfloat16*>(bias), iCout, iCin, iG,
            b.w_f32, b.bias_f32, b.w_f64, b.bias_f64);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "weight transform launch");
    if (b.img) {
        const size_t n = pl.img_alloc_bytes / 2;
        const unsigned b2 = static_cast<unsigned>((n + threads - 1) / threads);
        if (pl.tm()) {
            eqlin::eqlin_prep_image_k16_kernel<<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG, pl.nK, pl.rows, n,
                                                                        b.img);
        } else {
            eqlin::eqlin_prep_image_kernel<<<b2, threads, 0, st>>>(b.w_f32, iCout, iCin, iG, pl.nK, pl.rows, n,
                                                                    b.img);
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
            case 2: eqlin::eqlin_fwd_f32_kernel<2><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout); break;
            case 4: eqlin::eqlin_fwd_f32_kernel<4><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout); break;
            case 8: eqlin::eqlin_fwd_f32_kernel<8><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout); break;
            default: eqlin::eqlin_fwd_f32_kernel<16><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout); break;
        }
    } else {
        auto encode = tensor_map_encoder();
        if (!encode) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        CUtensorMap map, ymap;
        cuuint32_t estr[2] = {1, 1};
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(Cin * G), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(Cin * G * 2)};
        cuuint32_t boxdim[2] = {static_cast<cuuint32_t>(pl.box_elems), static_cast<cuuint32_t>(pl.BN)};
        CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, boxdim,
                            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
        cuuint64_t ydims[2] = {static_cast<cuuint64_t>(Cout * G), static_cast<cuuint64_t>(N)};
        cuuint64_t ystrides[1] = {static_cast<cuuint64_t>(Cout * G * 2)};
        cuuint32_t ybox[2];
        CUtensorMapSwizzle yswz;
        if (pl.tm()) {
            ybox[0] = eqlin::tm::kYCols;
            ybox[1] = eqlin::tm::kM;
            yswz = CU_TENSOR_MAP_SWIZZLE_64B;
        } else {
            ybox[0] = static_cast<cuuint32_t>(std::min<int64_t>(32 * G, eqlin::tc::kYBoxCols2));
            ybox[1] = static_cast<cuuint32_t>(pl.TG);
            yswz = CU_TENSOR_MAP_SWIZZLE_NONE;
        }
        r = encode(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, ydims, ystrides, ybox, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, yswz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for y");
        const long long n_tiles = (N + pl.BN - 1) / pl.BN;
        const int n_work = static_cast<int>(n_tiles * pl.n_oc);
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
            const TmEntry entry = tm_entry_for(iG, pl.streamed());
            if (!entry.launch) return fail(EQLIN_ERR_UNSUPPORTED, "G");
            entry.launch(grid, pl.smem_bytes, st, map, ymap, p);
        } else {
            TcParams p;
            p.w_img = b.img;
            p.bias = b.has_bias ? b.bias_f32 : nullptr;
            p.y = static_cast<__nv_bfloat16*>(y);
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
            p.w_img_bytes = pl.w_img_bytes;
            p.timeout_ns = timeout_ns;
            const TcEntry entry = tc_entry_for(iG, pl.streamed(), pl.nacc);
            if (!entry.launch) return fail(EQLIN_ERR_UNSUPPORTED, "G");
            entry.launch(grid, pl.smem_bytes, st, map, ymap, p);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return EQLIN_OK;
}

}  // namespace

struct eqlin_handle {
    int device = 0;
    int sm_count = 0;
    int64_t Cout = 0, Cin = 0, G = 0;
    int w_dtype = 0, io_dtype = 0;
    Plan plan;
    WeightBuffers buf;   // device memory owned by the handle
    bool sync_check = false;
    unsigned long long timeout_ns = kDefaultTimeoutNs;
};

namespace {

void free_handle(eqlin_handle* h) {
    if (!h) return;
    if (h->buf.img) cudaFree(h->buf.img);
    if (h->buf.w_f32) cudaFree(h->buf.w_f32);
    if (h->buf.bias_f32) cudaFree(h->buf.bias_f32);
    if (h->buf.w_f64) cudaFree(h->buf.w_f64);
    if (h->buf.bias_f64) cudaFree(h->buf.bias_f64);
    if (h->buf.status) cudaFree(h->buf.status);
    delete h;
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
    if (!out) return fail(EQLIN_ERR_INVALID_ARG, "out is NULL");
    *out = nullptr;
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
    e = cudaFuncSetAttribute(kernel_for(plan, static_cast<int>(G)), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(plan.smem_bytes));
    if (e != cudaSuccess) {
        free_handle(h);
        return cuda_fail(e, "cudaFuncSetAttribute");
    }
    *out = h;
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
    switch (attr) {
        case EQLIN_ATTR_G: *value = h->G; break;
        case EQLIN_ATTR_CIN: *value = h->Cin; break;
        case EQLIN_ATTR_COUT: *value = h->Cout; break;
        case EQLIN_ATTR_IO_DTYPE: *value = h->io_dtype; break;
        case EQLIN_ATTR_PATH: *value = pl.path; break;
        case EQLIN_ATTR_TOKENS_PER_TILE: *value = pl.BN; break;
        case EQLIN_ATTR_STAGES: *value = pl.stages; break;
        case EQLIN_ATTR_SMEM_BYTES: *value = static_cast<int64_t>(pl.smem_bytes); break;
        case EQLIN_ATTR_MAX_GRID: *value = pl.path == kPathF32 ? -1 : h->sm_count; break;
        case EQLIN_ATTR_WEIGHT_BYTES:
            *value = pl.path == kPathF32 ? static_cast<int64_t>(h->G * h->Cin * h->Cout * 8)
                                         : static_cast<int64_t>(pl.img_alloc_bytes);
            break;
        default: return fail(EQLIN_ERR_INVALID_ARG, "unknown attribute");
    }
    return EQLIN_OK;
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
constexpr int kNumPaths = 5;

struct NoAllocDevice {
    bool ready = false;
    uint8_t* scratch = nullptr;  // device address of g_noalloc_scratch on this device
    int sm_count = 0;
    int optin = 0;
    bool cc_ok = false;
    uint8_t attr_done[kNumPaths][4][2] = {};  // [path][G index][nacc-1]: smem attribute set
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
        // kernel shared-memory attribute, once per kernel and device
        uint8_t& done = d->attr_done[plan.path][g_index(G)][plan.nacc == 1 ? 0 : 1];
        if (!done) {
            e = cudaFuncSetAttribute(kernel_for(plan, static_cast<int>(G)),
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(plan.smem_bytes));
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
