// eqlin_host_mlp.h -- host side of the fused MLP block (eqlin_mlp_* in eqlin.h): planning,
// weight transforms and the launch (included once, by eqlin_api.cu, after
// eqlin_host_launch.h).
#pragma once

namespace {

constexpr int kMlpMaxStages = eqlin::mlp::kMaxStages;

struct MlpPlan {
    int io = EQLIN_BF16;
    int nK1 = 0, n_hc = 0, nK2 = 0, rows2 = 0;
    int BN = 0;              // tokens per tile (16-bit kernel)
    int stages = 0;          // weight ring depth (16-bit kernel)
    size_t smem_bytes = 0;
    size_t img1_bytes = 0, img2_bytes = 0;
    Plan layer1, layer2;     // for the weight transforms (launch_prep)
};

template <int G>
int plan_mlp_tc_g(int64_t Cin, int64_t H, int64_t Cout, size_t max_smem, MlpPlan* pl) {
    using S = eqlin::tc::Shape<G, 2>;
    if (Cout > eqlin::kMmaM) return fail(EQLIN_ERR_UNSUPPORTED, "the fused MLP block needs Cout <= 128");
    pl->nK1 = static_cast<int>((Cin + eqlin::kChunkK - 1) / eqlin::kChunkK);
    if (pl->nK1 > eqlin::mlp::kMaxK1) return fail(EQLIN_ERR_UNSUPPORTED, "the fused MLP block needs Cin <= 256");
    pl->n_hc = static_cast<int>((H + eqlin::kMmaM - 1) / eqlin::kMmaM);
    pl->nK2 = static_cast<int>((H + eqlin::kChunkK - 1) / eqlin::kChunkK);
    pl->rows2 = static_cast<int>((Cout + 7) / 8 * 8);
    pl->BN = S::BN;
    const size_t fixed = kSmemAlignSlack + kSmemCtlBytes + static_cast<size_t>(pl->nK1 + eqlin::mlp::kHK) * S::SPEC_BYTES;
    const int max_stages = std::min(kMlpMaxStages, env_int("EQLIN_MAX_STAGES", kMlpMaxStages));
    const size_t stages =
        max_smem > fixed ? std::min<size_t>(max_stages, (max_smem - fixed) / eqlin::mlp::kUnitBytes) : 0;
    if (stages < 2) return fail(EQLIN_ERR_UNSUPPORTED, "the fused MLP block does not fit in shared memory (Cin too large)");
    pl->stages = static_cast<int>(stages);
    pl->smem_bytes = fixed + stages * eqlin::mlp::kUnitBytes;
    // W1^ in the tokens-on-N image form with 128-row chunks of the hidden layer,
    // W2^ with one chunk of rows2 rows; both are read through the ring in units
    pl->img1_bytes = static_cast<size_t>(pl->n_hc) * pl->nK1 * G * eqlin::kMmaM * eqlin::kPlaneRowBytes;
    pl->img2_bytes = static_cast<size_t>(pl->nK2) * G * pl->rows2 * eqlin::kPlaneRowBytes;
    return EQLIN_OK;
}

int plan_mlp(int64_t Cin, int64_t H, int64_t Cout, int64_t G, int io, size_t max_smem, MlpPlan* pl) {
    int s = check_shape_impl(H, Cin, G, io, io);
    if (s == EQLIN_OK) s = check_shape_impl(Cout, H, G, io, io);
    if (s != EQLIN_OK) return s;
    pl->io = io;
    Plan l1, l2;
    l1.io = l2.io = io;
    if (io == EQLIN_F32) {
        const size_t smem = static_cast<size_t>(eqlin::kF32Tokens) * G * (Cin + H) * sizeof(double);
        if (smem > max_smem) return fail(EQLIN_ERR_UNSUPPORTED, "(Cin + H) * G too large for the fp32 MLP block");
        pl->smem_bytes = smem;
        pl->BN = eqlin::kF32Tokens;
        l1.path = l2.path = kPathF32;
    } else {
        switch (G) {
            case 2: s = plan_mlp_tc_g<2>(Cin, H, Cout, max_smem, pl); break;
            case 4: s = plan_mlp_tc_g<4>(Cin, H, Cout, max_smem, pl); break;
            case 8: s = plan_mlp_tc_g<8>(Cin, H, Cout, max_smem, pl); break;
            default: s = plan_mlp_tc_g<16>(Cin, H, Cout, max_smem, pl); break;
        }
        if (s != EQLIN_OK) return s;
        // image geometry for eqlin_prep_image_kernel (path 1: tokens-on-N image layout)
        l1.path = l2.path = kPathStreamed;
        l1.nK = pl->nK1;
        l1.rows = eqlin::kMmaM;
        l1.img_alloc_bytes = pl->img1_bytes;
        l2.nK = pl->nK2;
        l2.rows = pl->rows2;
        l2.img_alloc_bytes = pl->img2_bytes;
    }
    pl->layer1 = l1;
    pl->layer2 = l2;
    return EQLIN_OK;
}

void* mlp_kernel_for(int G, int io) {
    if (io == EQLIN_F32) {
        switch (G) {
            case 2: return reinterpret_cast<void*>(&eqlin::eqlin_mlp_f32_kernel<2>);
            case 4: return reinterpret_cast<void*>(&eqlin::eqlin_mlp_f32_kernel<4>);
            case 8: return reinterpret_cast<void*>(&eqlin::eqlin_mlp_f32_kernel<8>);
            default: return reinterpret_cast<void*>(&eqlin::eqlin_mlp_f32_kernel<16>);
        }
    }
    const bool f16 = io == EQLIN_F16;
    switch (G) {
        case 2: return f16 ? reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<2, __half>)
                           : reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<2, __nv_bfloat16>);
        case 4: return f16 ? reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<4, __half>)
                           : reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<4, __nv_bfloat16>);
        case 8: return f16 ? reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<8, __half>)
                           : reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<8, __nv_bfloat16>);
        default: return f16 ? reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<16, __half>)
                            : reinterpret_cast<void*>(&eqlin::eqlin_mlp_tc_kernel<16, __nv_bfloat16>);
    }
}

template <int G, class T16>
void mlp_tc_launch(unsigned grid, size_t smem, cudaStream_t st, const CUtensorMap& mx, const eqlin::MlpParams& p) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(eqlin::tc::kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = use_pdl() ? 1 : 0;
    cudaLaunchKernelEx(&cfg, eqlin::eqlin_mlp_tc_kernel<G, T16>, mx, p);
}

int launch_mlp(const MlpPlan& pl, int64_t Cin, int64_t H, int64_t Cout, int64_t G, int sm_count, const void* x,
               void* y, int64_t N, const WeightBuffers& b1, const WeightBuffers& b2, unsigned long long timeout_ns,
               cudaStream_t st) {
    const int iG = static_cast<int>(G), iCin = static_cast<int>(Cin), iH = static_cast<int>(H),
              iCout = static_cast<int>(Cout);
    if (pl.io == EQLIN_F32) {
        const unsigned grid = static_cast<unsigned>((N + eqlin::kF32Tokens - 1) / eqlin::kF32Tokens);
        const float* xf = static_cast<const float*>(x);
        float* yf = static_cast<float*>(y);
        const double* c1 = b1.has_bias ? b1.bias_f64 : nullptr;
        const double* c2 = b2.has_bias ? b2.bias_f64 : nullptr;
        switch (iG) {
            case 2: eqlin::eqlin_mlp_f32_kernel<2><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b1.w_f64, c1, b2.w_f64, c2, yf, N, iCin, iH, iCout); break;
            case 4: eqlin::eqlin_mlp_f32_kernel<4><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b1.w_f64, c1, b2.w_f64, c2, yf, N, iCin, iH, iCout); break;
            case 8: eqlin::eqlin_mlp_f32_kernel<8><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b1.w_f64, c1, b2.w_f64, c2, yf, N, iCin, iH, iCout); break;
            default: eqlin::eqlin_mlp_f32_kernel<16><<<grid, eqlin::kF32Threads, pl.smem_bytes, st>>>(xf, b1.w_f64, c1, b2.w_f64, c2, yf, N, iCin, iH, iCout); break;
        }
    } else {
        auto encode = tensor_map_encoder();
        if (!encode) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
        CUtensorMap map;
        cuuint32_t estr[2] = {1, 1};
        cuuint64_t dims[2] = {static_cast<cuuint64_t>(Cin * G), static_cast<cuuint64_t>(N)};
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(Cin * G * 2)};
        const int box_elems = static_cast<int>(std::min<int64_t>(eqlin::kChunkK * G, 256));
        cuuint32_t boxdim[2] = {static_cast<cuuint32_t>(box_elems), static_cast<cuuint32_t>(pl.BN)};
        CUresult r = encode(&map, pl.io == EQLIN_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                            2, const_cast<void*>(x), dims, strides, boxdim, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return fail(EQLIN_ERR_CUDA, "cuTensorMapEncodeTiled failed for x");
        eqlin::MlpParams p;
        p.w1_img = b1.img;
        p.w2_img = b2.img;
        p.b1 = b1.has_bias ? b1.bias_f32 : nullptr;
        p.b2 = b2.has_bias ? b2.bias_f32 : nullptr;
        p.y = static_cast<uint8_t*>(y);
        p.status = b1.status;
        p.N = N;
        p.Cin = iCin;
        p.H = iH;
        p.Cout = iCout;
        p.nK1 = pl.nK1;
        p.n_hc = pl.n_hc;
        p.nK2 = pl.nK2;
        p.rows2 = pl.rows2;
        p.n_tiles = static_cast<int>((N + pl.BN - 1) / pl.BN);
        p.stages = pl.stages;
        p.timeout_ns = timeout_ns;
        p.inject_stop = b1.inject_stop;
        p.w_early = (b1.w_early && b2.w_early) ? 1 : 0;
        p.pf = prefetch_distance();
        p.l2hint = l2_hint() ? 1 : 0;
        const unsigned grid = static_cast<unsigned>(std::min<long long>(p.n_tiles, sm_count));
        const bool f16 = pl.io == EQLIN_F16;
        switch (iG) {
            case 2: f16 ? mlp_tc_launch<2, __half>(grid, pl.smem_bytes, st, map, p)
                        : mlp_tc_launch<2, __nv_bfloat16>(grid, pl.smem_bytes, st, map, p); break;
            case 4: f16 ? mlp_tc_launch<4, __half>(grid, pl.smem_bytes, st, map, p)
                        : mlp_tc_launch<4, __nv_bfloat16>(grid, pl.smem_bytes, st, map, p); break;
            case 8: f16 ? mlp_tc_launch<8, __half>(grid, pl.smem_bytes, st, map, p)
                        : mlp_tc_launch<8, __nv_bfloat16>(grid, pl.smem_bytes, st, map, p); break;
            default: f16 ? mlp_tc_launch<16, __half>(grid, pl.smem_bytes, st, map, p)
                         : mlp_tc_launch<16, __nv_bfloat16>(grid, pl.smem_bytes, st, map, p); break;
        }
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "MLP block launch");
    return EQLIN_OK;
}

}  // namespace
