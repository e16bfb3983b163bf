// eqlin_host_launch.h -- kernel tables, TMA descriptors and launches of the forward, the
// weight pre-transform and the weight gradient (included once, by eqlin_api.cu, after
// eqlin_host_plan.h).
#pragma once

namespace {

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

// L2 eviction priorities on the fused kernels' copies (weights evict last, x and y evict
// first).  EQLIN_L2HINT=0 turns them off.
bool l2_hint() {
    static const bool on = [] {
        const char* e = std::getenv("EQLIN_L2HINT");
        return e && *e ? e[0] != '0' : kDefaultL2Hint;
    }();
    return on;
}

// L2 prefetch distance of the fused kernels' producer, in work items of the CTA.
// EQLIN_PREFETCH=k overrides (0 turns the prefetch off).
int prefetch_distance() {
    static const int d = [] {
        const char* e = std::getenv("EQLIN_PREFETCH");
        if (e && *e) {
            const int v = std::atoi(e);
            if (v >= 0 && v <= 16) return v;
        }
        return kDefaultPrefetch;
    }();
    return d;
}

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
    // The weights were complete before any forward using them was queued (a handle's:
    // prepare synchronises its stream), so the fused kernels may load them before
    // griddepcontrol.wait.  False for weights a kernel of the same stream writes just
    // before the forward (the allocation-free entry point's scratch).
    bool w_early = false;
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
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(eqlin::kF32Threads);
        cfg.dynamicSmemBytes = pl.smem_bytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = use_pdl() ? 1 : 0;
        cudaError_t e;
        switch (iG) {
            case 2: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_fwd_f32_kernel<2>, xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            case 4: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_fwd_f32_kernel<4>, xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            case 8: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_fwd_f32_kernel<8>, xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
            default: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_fwd_f32_kernel<16>, xf, b.w_f64, b.bias_f64, yf, N, iCin, iCout, b.act); break;
        }
        if (e != cudaSuccess) return cuda_fail(e, "fp32 forward launch");
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
            p.w_early = b.w_early ? 1 : 0;
            p.pf = prefetch_distance();
            p.l2hint = l2_hint() ? 1 : 0;
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
            p.yq = pl.yq;
            p.y = static_cast<uint8_t*>(y);
            p.w_img_bytes = pl.w_img_bytes;
            p.timeout_ns = timeout_ns;
            p.act = b.act;
            p.inject_stop = b.inject_stop;
            p.w_early = b.w_early ? 1 : 0;
            p.pf = prefetch_distance();
            p.l2hint = l2_hint() ? 1 : 0;
            const TcEntry entry = pl.tnr() ? tcr_entry_for(iG, pl.io) : tc_entry_for(iG, pl.streamed(), pl.nacc, pl.io);
            if (!entry.launch) return fail(EQLIN_ERR_UNSUPPORTED, "G");
            entry.launch(grid, pl.smem_bytes, st, map, ymap, p);
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "forward launch");
    return EQLIN_OK;
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
                    int io, CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    auto encode = tensor_map_encoder();
    if (!encode) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint32_t estr[2] = {1, 1};
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
    CUresult r = encode(map, io == EQLIN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
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
    const CUtensorMapSwizzle swz = iG == 2 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
    int s = encode_rows_map(&mdy, dy, Cout * G, N, pl.cpb_dy * iG, dw_tok(G), pl.io, swz);
    if (s != EQLIN_OK) return s;
    s = encode_rows_map(&mx, x, Cin * G, N, pl.cpb_x * iG, dw_tok(G), pl.io, swz);
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
    // a programmatic dependent of the main kernel (its blocks wait for the slabs)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(fgrid);
    cfg.blockDim = dim3(eqlin::kDwFinishWarps * 32);
    cfg.dynamicSmemBytes = static_cast<size_t>(eqlin::kDwFinishWarps) * iG * 32 * sizeof(double);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = use_pdl() ? 1 : 0;
    // 64 KB of warp sums at G = 16: above the default 48 KB, opted in on the current device
    if (iG == 16 && (e = cudaFuncSetAttribute(eqlin::eqlin_dw_finish_kernel<16>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                                              static_cast<int>(cfg.dynamicSmemBytes))) != cudaSuccess)
        return cuda_fail(e, "cudaFuncSetAttribute (weight-gradient reduction)");
    switch (iG) {
        case 2: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_dw_finish_kernel<2>, f); break;
        case 4: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_dw_finish_kernel<4>, f); break;
        case 8: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_dw_finish_kernel<8>, f); break;
        default: e = cudaLaunchKernelEx(&cfg, eqlin::eqlin_dw_finish_kernel<16>, f); break;
    }
    if (e != cudaSuccess) return cuda_fail(e, "weight-gradient reduction launch");
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_fail(e, "weight-gradient reduction launch");
    return EQLIN_OK;
}

}  // namespace
