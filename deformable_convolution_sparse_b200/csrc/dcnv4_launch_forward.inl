// Launcher of the forward aggregation: kernel choice, the tile kernel's planner
// (group subset, tile, halo, tensor map of x) and the dispatch over the
// kernels' template specialisations. Included by dcnv4.cu inside its anonymous
// namespace, after dcnv4_host_common.inl.

// Kernel choice: DCNV4_VARIANT=gather forces the global-gather kernel (A/B
// comparisons); unset or anything else selects the persistent shared-memory
// tile kernel whenever the shape allows it. DCNV4_HALO overrides the window
// halo (pixels) and DCNV4_TILE=<TH>x<TW> the output tile, for tuning runs.
enum class Variant { Auto, Gather };

Variant variant_from_env() {
    const char* v = std::getenv("DCNV4_VARIANT");
    if (v && std::strcmp(v, "gather") == 0) return Variant::Gather;
    return Variant::Auto;
}

// consumer threads (15 warps) per CTA, plus one producer warp: 16 warps, 4 per SM
// sub-partition, whose 16 K registers then hold 4 warps at the kernel's 112-register cap
// (a 17th warp would put 5 on one sub-partition: 17,920 registers, and the CTA would not launch)
constexpr int kTileUnitsMax = 480;
static_assert(((kTileUnitsMax / 32 + 1 + 3) / 4) * 112 * 32 <= 16384,
              "the tile kernel's register cap must fit the warps of one SM sub-partition");

// Mean shared-memory wavefronts of one quarter-warp LDS.128 in the tile
// kernel's gather, for window pixels of GS groups x Q chunks (PB = 16 GS Q
// bytes). A quarter warp is 8 consecutive units: ceil(8 / GS) pixels at
// independent window positions, each read at the lane's rotated chunk (the
// kernel's `rot`). With PB a multiple of 128 a chunk's bank quad does not depend
// on the pixel and the rotation makes it exactly 1; otherwise the pixels'
// placements collide on bank quads and the mean is taken over 256 placements
// drawn by a fixed linear congruential generator, so the plan stays
// deterministic. Cached per (Q, GS).
double gather_wavefronts(int Q, int GS) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, double> cache;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(Q, GS);
    if (auto it = cache.find(key); it != cache.end()) return it->second;
    const int step = GS * Q;  // chunks per pixel
    const int npx = GS < 8 ? (8 + GS - 1) / GS : 1;
    int rot[8];
    for (int l = 0; l < 8; ++l) rot[l] = Q == 2 ? (l >> 2) : Q == 4 ? (l >> 1) : Q == 8 ? l : 0;
    unsigned s = 12345u;
    double total = 0.0;
    long n = 0;
    for (int it = 0; it < 256; ++it) {
        long long pos[8];
        for (int p = 0; p < npx; ++p) {
            s = (s * 1103515245u + 12345u) & 0x7fffffffu;
            pos[p] = s >> 8;
        }
        for (int j = 0; j < Q; ++j) {
            long long addr[8];
            int cnt[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            for (int l = 0; l < 8; ++l) {
                const int gl = GS < 8 ? l % GS : l, p = GS < 8 ? l / GS : 0;
                addr[l] = pos[p] * step + gl * Q + (rot[l] + j) % Q;
                bool dup = false;
                for (int m = 0; m < l; ++m) dup = dup || addr[m] == addr[l];
                if (!dup) ++cnt[addr[l] % 8];
            }
            total += *std::max_element(cnt, cnt + 8);
            ++n;
        }
    }
    const double w = total / static_cast<double>(n);
    cache.emplace(key, w);
    return w;
}

struct TilePlan {
    dcnv4::TileParams p;
    CUtensorMap map;
    size_t smem;
    int threads;
};

// Chooses group subset, tile and halo for the tile kernel and encodes the
// tensor map of x; false when the shape or the alignment does not suit it.
template <typename T>
bool plan_tile(const void* x, const void* om, const void* out, const FwdParams& f, TilePlan* plan) {
    constexpr int E = sizeof(T);
    const int row_bytes = f.Cg * E;
    if (!aligned(x, 16) || !aligned(out, 16) || (f.C * E) % 16 || row_bytes % 16) return false;
    const int Q = row_bytes / 16;
    if (!(Q == 1 || Q == 2 || Q == 4 || Q == 5 || Q == 8)) return false;
    if (f.KK > 64) return false;  // the per-unit mask of points outside the window has 64 bits
    int R = 5;
    if (const char* h = std::getenv("DCNV4_HALO")) R = std::atoi(h) > 0 ? std::atoi(h) : R;
    int forceTH = 0, forceTW = 0, forceGS = 0, forceNrec = 0;
    if (const char* n = std::getenv("DCNV4_NREC")) forceNrec = (std::atoi(n) == 2 || std::atoi(n) == 3) ? std::atoi(n) : 0;
    if (const char* t = std::getenv("DCNV4_TILE")) std::sscanf(t, "%dx%d", &forceTH, &forceTW);
    if (const char* g = std::getenv("DCNV4_GS")) forceGS = std::atoi(g);
    const int R3 = 3 * f.npts;
    const int nsm = sm_count();
    if (nsm <= 0) return false;

    static const int THs[] = {1, 2, 4, 7, 8, 14, 16, 28, 32};
    static const int TWs[] = {1, 2, 4, 7, 8, 14, 16, 28, 32};
    double best = -1.0;
    dcnv4::TileParams bp{};
    int best_threads = 0, best_c2 = 0;
    size_t best_smem = 0;
    for (int GS = 1; GS <= f.G; ++GS) {
        if (f.G % GS || (forceGS && GS != forceGS)) continue;
        const int PB = GS * row_bytes;
        const int sub_ch = GS * f.Cg;
        int c2 = 0;
        for (int d = std::min(sub_ch, 256); d >= 1; --d)
            if (sub_ch % d == 0 && (d * E) % 16 == 0) { c2 = d; break; }
        if (c2 == 0 || sub_ch / c2 > 256) continue;
        // a pixel stride that is a multiple of 128 bytes keeps the gathers free of
        // bank conflicts (see the kernel); other strides pay in extra wavefronts.
        // The gather's shared-memory reads dominate a tile's cost there, and the
        // squared factor matches the measured 1.21x between 80- and 160-byte
        // pixels of the 40-channel groups (2.60 vs 2.13 wavefronts), against
        // which the window-reuse and ring-depth terms would otherwise win.
        const double w = gather_wavefronts(Q, GS);
        const double banks = 1.0 / (w * w);
        const bool row_runs = GS == f.G;
        for (int TH : THs) {
            for (int TW : TWs) {
                if (forceTH && (TH != forceTH || TW != forceTW)) continue;
                const int units = TH * TW * GS;
                if (units > kTileUnitsMax || units < 32) continue;
                if (TH > f.Hout + 7 || TW > f.Wout + 7) continue;
                const int WH = (TH - 1) * f.stride + (f.K - 1) * f.dilation + 2 * R + 1;
                const int WW = (TW - 1) * f.stride + (f.K - 1) * f.dilation + 2 * R + 1;
                if (WH > 256 || WW > 256) continue;
                const int nruns = row_runs ? TH : TH * TW;
                const int count = (row_runs ? TW * f.G : GS) * R3;
                const int slot = (count * E + 32 + 15) / 16 * 16;
                const size_t rec = (static_cast<size_t>(nruns) * slot + 127) / 128 * 128;
                const size_t win = (static_cast<size_t>(WH) * WW * PB + 127) / 128 * 128;
                // records get a third buffer (a longer lead for their DRAM reads) when it fits
                int nrec = (2 * win + 3 * rec <= kTileSmemLimit) ? 3 : 2;
                if (forceNrec) nrec = forceNrec;
                const size_t smem = 2 * win + nrec * rec;
                if (smem > kTileSmemLimit) continue;
                const int threads = (units + 31) / 32 * 32 + 32;  // consumers + the producer warp
                const int tiles_y = (f.Hout + TH - 1) / TH, tiles_x = (f.Wout + TW - 1) / TW;
                const long long tiles = static_cast<long long>(f.N) * tiles_y * tiles_x * (f.G / GS);
                // the choice must not depend on N: an image's result (which samples take
                // the window path) then never depends on the batch it comes in. The wave
                // balance is judged for a nominal batch of 64 images.
                const long long tiles_nominal = 64LL * tiles_y * tiles_x * (f.G / GS);
                const int per_sm = std::max(1, static_cast<int>(std::min<size_t>(
                                                   (kTileSmemLimit + 2048) / (smem + 1024), 2048 / threads)));
                const double slots = static_cast<double>(nsm) * per_sm;
                const double waves = static_cast<double>(tiles_nominal) / slots;
                const double balance = waves / std::ceil(waves);
                const double useful =
                    static_cast<double>(f.Hout) * f.Wout / (static_cast<double>(tiles_y) * TH * tiles_x * TW);
                const double reuse = static_cast<double>(TH * TW) / (static_cast<double>(WH) * WW);
                const double fill = static_cast<double>(units) / (threads - 32);
                const double occ = std::min(1.0, per_sm * (threads - 32) / 384.0);
                const double depth = nrec == 3 ? 1.0 : 0.9;
                // a ragged tile loses threads and still loads a full window: useful counts twice
                const double score = useful * useful * balance * fill * occ * banks * depth * std::sqrt(reuse);
                if (score > best) {
                    best = score;
                    bp.TH = TH; bp.TW = TW; bp.tiles_x = tiles_x; bp.tiles_y = tiles_y;
                    bp.WH = WH; bp.WW = WW; bp.run_slot = slot; bp.rec_bytes = static_cast<int>(rec);
                    bp.win_bytes = static_cast<int>(win);
                    bp.nrec = nrec;
                    bp.tiles = static_cast<int>(tiles); bp.units = units;
                    bp.GS = GS; bp.PB = PB; bp.cblk = sub_ch / c2;
                    best_threads = threads;
                    best_smem = smem;
                    best_c2 = c2;
                }
            }
        }
    }
    if (best < 0) return false;
    const int GS = bp.GS, PB = bp.PB, c2 = best_c2;
    bp.f = f;
    bp.nsub = f.G / GS;
    bp.R = R;
    const size_t om_bytes = static_cast<size_t>(f.N) * f.Hout * f.Wout * f.G * R3 * E;
    bp.om_lo = reinterpret_cast<unsigned long long>(om);
    bp.om_hi = bp.om_lo + om_bytes;
    bp.div_tw_gs = dcnv4::make_fastdiv(bp.TW * GS);
    bp.div_gs = dcnv4::make_fastdiv(GS);
    bp.div_nsub = dcnv4::make_fastdiv(bp.nsub);
    bp.div_tx = dcnv4::make_fastdiv(bp.tiles_x);
    bp.div_ty = dcnv4::make_fastdiv(bp.tiles_y);

    auto encode = tensor_map_encoder();
    if (!encode) return false;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(c2), static_cast<cuuint64_t>(f.C / c2),
                                static_cast<cuuint64_t>(f.W), static_cast<cuuint64_t>(f.H),
                                static_cast<cuuint64_t>(f.N)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(c2) * E, static_cast<cuuint64_t>(f.C) * E,
                                   static_cast<cuuint64_t>(f.W) * f.C * E,
                                   static_cast<cuuint64_t>(f.H) * f.W * f.C * E};
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(c2), static_cast<cuuint32_t>(bp.cblk),
                               static_cast<cuuint32_t>(bp.WW), static_cast<cuuint32_t>(bp.WH), 1u};
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    if (encode(&plan->map, tma_dtype<T>(), 5, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    plan->p = bp;
    plan->smem = best_smem;
    plan->threads = best_threads;
    if (const char* d = std::getenv("DCNV4_DEBUG"); d && *d == '1')
        std::fprintf(stderr,
                     "dcnv4 tile plan: tile %dx%d GS %d (nsub %d) R %d window %dx%d PB %d cblk %d tiles %d units %d "
                     "threads %d nrec %d smem %zu\n",
                     bp.TH, bp.TW, GS, bp.nsub, R, bp.WH, bp.WW, PB, bp.cblk, bp.tiles, bp.units, best_threads,
                     bp.nrec, best_smem);
    return true;
}

// fp16 storage: weights rounded to fp16 for the mixed-precision FMA (default)
// or kept in fp32 (DCNV4_F16_EXACT=1, for comparisons).
bool f16_exact_from_env() {
    const char* v = std::getenv("DCNV4_F16_EXACT");
    return v && *v == '1';
}

template <typename T, int Q, int KS, bool HW, int PBC, bool VF = false>
int launch_tile_q(const T* x, const T* om, T* out, const TilePlan& plan, cudaStream_t stream) {
    auto kern = dcnv4::fwd_tile_kernel<T, Q, KS, HW, PBC, VF>;
    static std::once_flag once;
    static cudaError_t attr = cudaSuccess;
    std::call_once(once, [&] {
        attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kTileSmemLimit));
    });
    const bool dbg = std::getenv("DCNV4_DEBUG") != nullptr;
    if (attr != cudaSuccess) {
        if (dbg) std::fprintf(stderr, "dcnv4 tile launch: shared-memory attribute: %s\n", cudaGetErrorString(attr));
        return DCNV4_ERR_LAUNCH;
    }
    int per_sm = 0;
    const cudaError_t occ = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, plan.threads, plan.smem);
    if (occ != cudaSuccess || per_sm < 1) {
        if (dbg) std::fprintf(stderr, "dcnv4 tile launch: occupancy %d (%s) for %d threads, %zu bytes\n", per_sm,
                              cudaGetErrorString(occ), plan.threads, plan.smem);
        return DCNV4_ERR_LAUNCH;
    }
    const long long slots = static_cast<long long>(sm_count()) * per_sm;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(plan.p.tiles, slots));
    // the last partial wave (tiles mod grid) is split by consumer warps over up to grid / L
    // CTAs when at least two can share each tile (DCNV4_TAIL_SPLIT=0 turns it off)
    dcnv4::TileParams p = plan.p;
    const int L = static_cast<int>(p.tiles % static_cast<int>(grid));
    const int consumer_warps = plan.threads / 32 - 1;
    int split = 1;
    if (L > 0 && static_cast<int>(grid) >= 2 * L) split = std::min(static_cast<int>(grid) / L, consumer_warps);
    if (const char* e = std::getenv("DCNV4_TAIL_SPLIT"); e && *e == '0') split = 1;
    p.tail_split = split;
    p.main_tiles = split > 1 ? p.tiles - L : p.tiles;
    p.items = p.main_tiles + (split > 1 ? L * split : 0);
    kern<<<grid, plan.threads, plan.smem, stream>>>(plan.map, x, om, out, p);
    const cudaError_t le = cudaGetLastError();
    if (le != cudaSuccess && dbg) std::fprintf(stderr, "dcnv4 tile launch: %s\n", cudaGetErrorString(le));
    return le == cudaSuccess ? DCNV4_OK : DCNV4_ERR_LAUNCH;
}

template <typename T, int Q, bool HW, bool VF>
int launch_tile_v(const T* x, const T* om, T* out, const TilePlan& plan, cudaStream_t s) {
    // a 128-byte window pixel (the common case) as a compile-time stride
    if constexpr (Q != 5) {
        if (plan.p.PB == 128) {
            if (plan.p.f.K == 3) return launch_tile_q<T, Q, 3, HW, 128, VF>(x, om, out, plan, s);
            return launch_tile_q<T, Q, 0, HW, 128, VF>(x, om, out, plan, s);
        }
    }
    if (plan.p.f.K == 3) return launch_tile_q<T, Q, 3, HW, 0, VF>(x, om, out, plan, s);
    return launch_tile_q<T, Q, 0, HW, 0, VF>(x, om, out, plan, s);
}

template <typename T, int Q, bool HW>
int launch_tile_k(const T* x, const T* om, T* out, const TilePlan& plan, cudaStream_t s) {
    // the variant flags get their own instantiations, so that the plain forward carries none of their code
    if (plan.p.f.flags != 0) return launch_tile_v<T, Q, HW, true>(x, om, out, plan, s);
    return launch_tile_v<T, Q, HW, false>(x, om, out, plan, s);
}

template <typename T, int Q>
int launch_tile_k(const T* x, const T* om, T* out, const TilePlan& plan, cudaStream_t s) {
    if constexpr (std::is_same<T, __half>::value) {
        if (!f16_exact_from_env()) return launch_tile_k<T, Q, true>(x, om, out, plan, s);
    }
    return launch_tile_k<T, Q, false>(x, om, out, plan, s);
}

template <typename T>
int launch_tile(const void* x, const void* om, void* out, const TilePlan& plan, cudaStream_t s) {
    const T* xt = static_cast<const T*>(x);
    const T* omt = static_cast<const T*>(om);
    T* ot = static_cast<T*>(out);
    switch (plan.p.f.Cg * static_cast<int>(sizeof(T)) / 16) {
        case 1: return launch_tile_k<T, 1>(xt, omt, ot, plan, s);
        case 2: return launch_tile_k<T, 2>(xt, omt, ot, plan, s);
        case 4: return launch_tile_k<T, 4>(xt, omt, ot, plan, s);
        case 5: return launch_tile_k<T, 5>(xt, omt, ot, plan, s);
        default: return launch_tile_k<T, 8>(xt, omt, ot, plan, s);
    }
}

// The global-gather kernels for one thread-slice width (lane_bytes: 64, 32 or
// 16 bytes per thread, 0 for the element-wise kernel).
template <typename T, bool VF>
int launch_gather(const T* xt, const T* omt, T* ot, const FwdParams& p, int lane_bytes, dim3 grid, int threads,
                  size_t smem, cudaStream_t stream) {
    const bool k3 = p.K == 3;
    if (lane_bytes == 64) {
        if (k3) dcnv4::fwd_vector_kernel<T, 32, 64, 3, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 32, 64, 0, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else if (lane_bytes == 32) {
        if (k3) dcnv4::fwd_vector_kernel<T, 32, 32, 3, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 32, 32, 0, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else if (lane_bytes == 16) {
        if (k3) dcnv4::fwd_vector_kernel<T, 16, 16, 3, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 16, 16, 0, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else {
        if (k3) dcnv4::fwd_scalar_kernel<T, 3, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_scalar_kernel<T, 0, VF><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    }
    return launch_status();
}

template <typename T>
int launch_forward(const void* x, const void* om, void* out, FwdParams p, cudaStream_t stream) {
    constexpr int E = sizeof(T);
    if (variant_from_env() == Variant::Auto) {
        TilePlan plan;
        if (plan_tile<T>(x, om, out, p, &plan)) return launch_tile<T>(x, om, out, plan, stream);
    }
    const int row_bytes = p.Cg * E;
    const bool a16 = aligned(x, 16) && aligned(out, 16) && (p.C * E) % 16 == 0;
    const bool a32 = aligned(x, 32) && aligned(out, 32) && (p.C * E) % 32 == 0;
    const size_t rec_bytes = static_cast<size_t>(3) * p.npts * E;

    int lane_bytes = 0, vec_bytes = 0;
    if (a16 && row_bytes % 16 == 0) {
        if (a32 && row_bytes % 32 == 0) {
            vec_bytes = 32;
            lane_bytes = (E == 4 && row_bytes % 64 == 0) ? 64 : 32;
        } else {
            vec_bytes = 16;
            lane_bytes = 16;
        }
    }
    if (lane_bytes) {
        p.chunks = row_bytes / lane_bytes;
        p.lanes = p.chunks < kThreads ? p.chunks : kThreads;
    } else {
        p.chunks = p.Cg;
        p.lanes = p.Cg < kThreads ? p.Cg : kThreads;
    }
    int upb = kThreads / p.lanes;
    const size_t smem_cap = 40 * 1024;
    while (upb > 1 && upb * rec_bytes + 16 > smem_cap) --upb;
    p.units_per_block = upb;
    const size_t smem = upb * rec_bytes + 16;
    const int threads = upb * p.lanes;
    const long long blocks = (static_cast<long long>(p.units) + upb - 1) / upb;
    if (blocks > 0x7fffffffLL) return DCNV4_ERR_TOO_LARGE;
    const dim3 grid(static_cast<unsigned>(blocks));

    const T* xt = static_cast<const T*>(x);
    const T* omt = static_cast<const T*>(om);
    T* ot = static_cast<T*>(out);
    // the variant flags get their own instantiations, as in the tile kernel
    if (p.flags != 0) return launch_gather<T, true>(xt, omt, ot, p, lane_bytes, grid, threads, smem, stream);
    return launch_gather<T, false>(xt, omt, ot, p, lane_bytes, grid, threads, smem, stream);
}
