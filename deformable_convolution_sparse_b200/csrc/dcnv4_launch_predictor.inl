// Launcher of the offset/mask predictor. Included by dcnv4.cu inside its
// anonymous namespace, after dcnv4_host_common.inl.
// Offset/mask predictor: the tensor-core kernel for fp16/bf16 with C a multiple
// of 64 and at most 256 output channels (DCNV4_PRED_VARIANT=plain forces the
// CUDA-core kernel), the CUDA-core kernel otherwise.
template <typename T>
int launch_predictor(const void* y, const void* w, const float* bias, void* rec, dcnv4::PredParams p,
                     cudaStream_t stream) {
    constexpr int E = sizeof(T);
    const char* pv = std::getenv("DCNV4_PRED_VARIANT");
    const bool force_plain = pv && std::strcmp(pv, "plain") == 0;
    bool tc = !force_plain && E == 2 && p.C % 64 == 0 && p.NO <= 256 && aligned(y, 16) && aligned(w, 16) &&
              aligned(rec, 16) && p.M > 0;
    if constexpr (E == 2) {
        if (tc) {
            p.NP = (p.NO + 15) / 16 * 16;
            p.kblocks = p.C / 64;
            p.tiles = (p.M + 127) / 128;
            // two accumulator buffers: the MMA runs one tile ahead of the epilogue (a third measured slower)
            unsigned cols = 32;
            while (cols < 2u * static_cast<unsigned>(p.NP)) cols <<= 1;
            p.tmem_cols = cols;
            p.a_fmt = std::is_same<T, __half>::value ? 0 : 1;
            const size_t b_bytes = static_cast<size_t>(p.kblocks) * p.NP * 128;
            const size_t a_stage = static_cast<size_t>(p.kblocks) * 128 * 128;
            constexpr int kMaxStages = 8;
            const size_t meta = static_cast<size_t>(p.NO) * 8 + 8 + 8 * (2 * kMaxStages + 1 + 2 * 2) + 16;
            // two output staging buffers (store of tile i overlaps the epilogue of tile i+1) when they fit
            size_t o_bytes = 0, fixed = 0;
            int stages = 0;
            for (int ob = 2; ob >= 1 && stages < 2; --ob) {
                o_bytes = (static_cast<size_t>(ob) * 128 * p.NO * E + 15) / 16 * 16;
                fixed = 1024 + b_bytes + o_bytes + meta;
                // 4 activation stages (6 and 8 measured no faster); DCNV4_PRED_STAGES overrides, up to 8
                stages = 4;
                if (const char* e = std::getenv("DCNV4_PRED_STAGES")) stages = std::min(kMaxStages, std::max(2, std::atoi(e)));
                while (stages >= 2 && fixed + stages * a_stage > kTileSmemLimit) --stages;
                p.out_bufs = ob;
            }
            tc = stages >= 2;
            if (tc) {
                p.stages = stages;
                // raw W in the staging area when it fits (DCNV4_PRED_WSTAGE=0 keeps it in the ring)
                p.w_in_staging = b_bytes <= o_bytes ? 1 : 0;
                if (const char* e = std::getenv("DCNV4_PRED_WSTAGE"); e && *e == '0') p.w_in_staging = 0;
                p.smem_b = 0;
                p.smem_a = static_cast<unsigned>(b_bytes);
                p.smem_o = static_cast<unsigned>(b_bytes + stages * a_stage);
                p.smem_meta = static_cast<unsigned>(p.smem_o + o_bytes);
                const size_t smem = fixed + stages * a_stage;
                auto encode = tensor_map_encoder();
                CUtensorMap amap, bmap;
                const cuuint32_t estr[2] = {1u, 1u};
                const cuuint64_t adims[2] = {static_cast<cuuint64_t>(p.C), static_cast<cuuint64_t>(p.M)};
                const cuuint64_t astr[1] = {static_cast<cuuint64_t>(p.C) * E};
                const cuuint32_t abox[2] = {64u, 128u};
                const cuuint64_t bdims[2] = {static_cast<cuuint64_t>(p.C), static_cast<cuuint64_t>(p.NO)};
                const cuuint32_t bbox[2] = {64u, static_cast<cuuint32_t>(p.NP)};
                tc = encode &&
                     encode(&amap, tma_dtype<T>(), 2, const_cast<void*>(y), adims, astr, abox, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
                     encode(&bmap, tma_dtype<T>(), 2, const_cast<void*>(w), bdims, astr, bbox, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
                if (tc) {
                    // epilogue warps: DCNV4_PRED_EPI=8 or 16 (tuning runs); default 16
                    int epw = 16;
                    if (const char* e = std::getenv("DCNV4_PRED_EPI")) epw = std::atoi(e) == 8 ? 8 : 16;
                    auto kern = epw == 8 ? dcnv4::predictor_tc_kernel<T, 8> : dcnv4::predictor_tc_kernel<T, 16>;
                    const int threads = 64 + 32 * epw;
                    if (smem_limit_once(reinterpret_cast<const void*>(kern), static_cast<int>(kTileSmemLimit)) !=
                        cudaSuccess)
                        return DCNV4_ERR_LAUNCH;
                    const int nsm = sm_count();
                    if (nsm <= 0) return DCNV4_ERR_CUDA;
                    const unsigned grid = static_cast<unsigned>(std::min(p.tiles, nsm));
                    if (std::getenv("DCNV4_DEBUG"))
                        std::fprintf(stderr, "dcnv4 predictor: tcgen05 NP %d kblocks %d stages %d out bufs %d tiles %d "
                                     "grid %u smem %zu tmem cols %u epilogue warps %d\n", p.NP, p.kblocks, p.stages,
                                     p.out_bufs, p.tiles, grid, smem, p.tmem_cols, epw);
                    // programmatic stream serialisation, as for the forward (DCNV4_PDL=0: plain)
                    cudaLaunchConfig_t cfg{};
                    cfg.gridDim = dim3(grid);
                    cfg.blockDim = dim3(static_cast<unsigned>(threads));
                    cfg.dynamicSmemBytes = smem;
                    cfg.stream = stream;
                    cudaLaunchAttribute pdl[1];
                    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
                    pdl[0].val.programmaticStreamSerializationAllowed = 1;
                    cfg.attrs = pdl;
                    const char* pe = std::getenv("DCNV4_PDL");
                    cfg.numAttrs = (pe && *pe == '0') ? 0 : 1;
                    if (cudaLaunchKernelEx(&cfg, kern, amap, bmap, bias, static_cast<T*>(rec), p) != cudaSuccess)
                        return DCNV4_ERR_LAUNCH;
                    return launch_status();
                }
            }
        }
    }
    // 8 warps per block, 4 pixels per warp
    const long long wblocks = (static_cast<long long>(p.M) + 31) / 32;
    const unsigned blocks = static_cast<unsigned>(std::min<long long>(wblocks, 148LL * 8));
    dcnv4::predictor_plain_kernel<T><<<blocks, 256, 0, stream>>>(
        static_cast<const T*>(y), static_cast<const T*>(w), bias, static_cast<T*>(rec), p);
    return launch_status();
}
