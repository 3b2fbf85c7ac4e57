// Launcher of the forward aggregation: kernel choice, the ring kernel's planner
// (group subset, band width, item height, halo, ring depth, tensor map of x)
// and the dispatch over the kernels' template specialisations. Included by the
// per-storage-type translation units (dcnv4_fwd_*.cu) inside their anonymous
// namespace, after dcnv4_host_common.inl.

// Kernel choice: DCNV4_VARIANT=gather forces the global-gather kernel (A/B
// comparisons); unset or anything else selects the ring kernel whenever the
// shape allows it. Tuning overrides of the planner: DCNV4_HALO (pixels),
// DCNV4_TILE=<TH>x<TW> (item rows x band columns), DCNV4_GS (groups per
// strip), DCNV4_NREC (items in flight, 2..4), DCNV4_RING (ring rows).
enum class Variant { Auto, Gather };

Variant variant_from_env() {
    const char* v = std::getenv("DCNV4_VARIANT");
    if (v && std::strcmp(v, "gather") == 0) return Variant::Gather;
    return Variant::Auto;
}

int env_int(const char* name, int dflt) {
    const char* v = std::getenv(name);
    return (v && *v) ? std::atoi(v) : dflt;
}

// consumer threads (15 warps) per CTA, plus one producer warp: 16 warps, 4 per SM
// sub-partition, whose 16 K registers then hold 4 warps at the kernel's 112-register cap
// (a 17th warp would put 5 on one sub-partition: 17,920 registers, and the CTA would not launch)
#ifndef DCNV4_RING_UNITS_MAX
#define DCNV4_RING_UNITS_MAX 480  // consumer threads per CTA (build option, with DCNV4_RING_MAXREG)
#endif
constexpr int kUnitsMax = DCNV4_RING_UNITS_MAX;
static_assert(((kUnitsMax / 32 + 1 + 3) / 4) * DCNV4_RING_MAXREG * 32 <= 16384 &&
                  ((kUnitsMax / 32 + 1 + 3) / 4) * DCNV4_RING_MAXREG_NARROW * 32 <= 16384,
              "the ring kernel's register cap must fit the warps of one SM sub-partition");

// Mean shared-memory wavefronts of one quarter-warp LDS.128 in the ring
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

// Smallest odd multiple of 16 that holds `bytes`: consecutive record slots
// then start on different 16-byte bank positions, so the record reads of a
// warp's pixels do not all fall on the same banks.
int odd16(int bytes) {
    int s = (bytes + 15) / 16;
    if ((s & 1) == 0) ++s;
    return s * 16;
}

// The halo the planner aims for: samples whose corners stay within R pixels of
// their unit's grid footprint are gathered from shared memory, so R bounds the
// offsets served from the window. The target R = 4*dilation + 1 serves every
// offset of up to four grid spacings (|d| <= 4*dilation: floor(d) + 1 <= R);
// the planner considers one pixel less and one more (see plan_ring).
int target_halo(int dilation) { return std::min(15, 4 * dilation + 1); }

// Image windows need the whole image plus a one-pixel border within one TMA
// row load (at most 256 pixels) and, for centre feature scaling, every unit's
// centre grid position inside that border (the kernel reads the centre pixel
// from the window).
bool image_window_fits(const FwdParams& f) {
    if (f.W + 2 > 256) return false;
    if (f.flags & dcnv4::kFlagCenterScale) {
        const int c = (f.K / 2) * f.dilation - f.pad;
        if (c < -1 || (f.Hout - 1) * f.stride + c > f.H || (f.Wout - 1) * f.stride + c > f.W) return false;
    }
    return true;
}

struct RingPlan {
    dcnv4::RingParams p;
    CUtensorMap map;
    size_t smem;
    int threads;
};

struct RingShape {  // one candidate of the planner
    int GS, R, TW, TH, nrec, NR, units, threads, slot, rec, WW, UH, UW, c2, img;
    size_t smem;
    double score;
    double row_us, strip_us;  // estimated time of one output row (band x groups) and of a strip's window load
};

// The best plan for halo R, or with image windows when `img` (score < 0: none
// fits), with at least `min_units` consumer threads. Everything but R and the
// window kind leaves the per-unit arithmetic unchanged; it is chosen for speed
// and may depend on N. An image window is the whole image plus a one-pixel
// border (H + 2 rows of W + 2 pixels), one band of all Wout columns, loaded
// once per strip. The score is the inverse of an estimated launch time
// (microseconds at 1.9 GHz), the sum of
//  - compute: a CTA's rows x band width x groups x points at (0.75*Q + 0.5)
//    SM cycles per sampling point (the measured rate of the 128-byte-pixel
//    gather), divided by the gather's bank efficiency (1 / wavefronts^2), the
//    record layout (per-pixel runs measured about 20 % slower than one run per
//    output row, except in image-window plans of 8 or more groups), warp occupancy (below 12 consumer warps, 8 with four or more
//    chunks per group), the filled lanes of
//    the consumer warps and bands narrower
//    than half their window (measured slower: (2 TW stride / WW)^(1/4));
//  - start-up: every CTA loads its first window and records at once, from HBM
//    at about 6.5 TB/s;
//  - strip changes that the ring cannot prefetch (NR < 2*nrows): about 1 us
//    plus the window's bytes at 100 B per cycle each, one per Hout rows of a
//    CTA's range;
//  - items whose rows cannot load during the previous item (NR < nrows +
//    TH*stride): about 1 us each.
template <typename T>
RingShape best_ring_shape(const FwdParams& f, int R, int nsm, int min_units, bool img = false) {
    constexpr int E = sizeof(T);
    const int row_bytes = f.Cg * E;
    const int Q = row_bytes / 16;
    const int R3 = 3 * f.npts;
    int forceTH = 0, forceTW = 0;
    if (const char* t = std::getenv("DCNV4_TILE")) std::sscanf(t, "%dx%d", &forceTH, &forceTW);
    const int forceGS = env_int("DCNV4_GS", 0);
    const int forceNrec = env_int("DCNV4_NREC", 0);
    const int forceNR = env_int("DCNV4_RING", 0);
    const int s = f.stride;
    const int UH = img ? f.H + 2 : (f.K - 1) * f.dilation + 2 * R + 1;
    const int UW = img ? f.W + 2 : UH;
    const double clk = 1.9e3;  // SM cycles per microsecond
    RingShape best{};
    best.score = -1.0;
    static const int TWs[] = {1, 2, 4, 7, 8, 14, 16, 28, 32, 56, 64};
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
        // The squared factor matches the measured 1.21x between 80- and 160-byte
        // pixels of the 40-channel groups (2.60 vs 2.13 wavefronts).
        const double w = gather_wavefronts(Q, GS);
        const double banks = 1.0 / (w * w);
        const bool row_runs = GS == f.G;
        // per-pixel record runs: 20 % slower in unit-window plans; image-window plans of 8 or more
        // groups per strip measured as fast as the row-run plan or faster (stage-3 shape: 8 groups
        // in 4-row items 17.2 us against 18.4 for all 16 groups in 2-row items)
        const double runs = (row_runs || (img && GS >= 8)) ? 1.0 : 0.8;
        for (int TW : TWs) {
            if (img) {
                if (TW != TWs[0]) break;
                TW = f.Wout;  // one band
            }
            if (forceTW && TW != forceTW) continue;
            if (!img && TW > f.Wout && TW != TWs[0]) {
                // one band wider than the image only if no narrower TW covers it
                bool smaller = false;
                for (int t2 : TWs) smaller = smaller || (t2 < TW && t2 >= f.Wout);
                if (smaller) continue;
            }
            const int WW = img ? UW : (TW - 1) * s + UW;
            if (WW > 256) continue;
            const int rowB = (WW * PB + 127) / 128 * 128;  // ring row pitch: every TMA destination 128-byte aligned
            const int bands = (f.Wout + TW - 1) / TW;
            const double rows_per_cta =
                static_cast<double>(f.N) * bands * (f.G / GS) * f.Hout / std::max(1, nsm);
            for (int TH = 1; TH <= 16; ++TH) {
                if (forceTH && TH != forceTH) continue;
                if (TH > f.Hout) break;
                const int units = TH * TW * GS;
                if (units > kUnitsMax) break;
                if (units < min_units) continue;
                const int nrows = img ? UH : (TH - 1) * s + UH;
                const int slot = odd16((row_runs ? TW * f.G : GS) * R3 * E + 32);
                const int rec = ((row_runs ? TH : TH * TW) * slot + 127) / 128 * 128;
                for (int nrec = 2; nrec <= 4; ++nrec) {
                    if (forceNrec ? nrec != forceNrec : nrec == 4) continue;
                    const long long avail = static_cast<long long>(kTileSmemLimit) - static_cast<long long>(nrec) * rec;
                    if (avail <= 0) continue;
                    int NR = static_cast<int>(avail / rowB) - 1;  // one mirror row
                    NR = std::min(NR, 2 * nrows);                 // deeper never helps
                    if (forceNR) NR = std::min(NR, forceNR);
                    if (NR < nrows) continue;
                    const size_t smem = (static_cast<size_t>(NR + 1) * rowB + 127) / 128 * 128 +
                                        static_cast<size_t>(nrec) * rec;
                    if (smem > kTileSmemLimit) continue;
                    const int threads = (units + 31) / 32 * 32 + 32;
                    const double warps = (threads - 32) / 32.0;
                    const double occ = std::min(1.0, warps / (Q >= 4 ? 8.0 : 12.0));  // fewer loads per point want more warps
                    // bands narrower than half their window (WW > 2 TW stride) measured slower
                    const double narrow = std::sqrt(std::sqrt(std::min(1.0, 2.0 * TW * s / WW)));
                    const double lanes = static_cast<double>(units) / (threads - 32);  // filled lanes of the last warp
                    const double cpp = (0.75 * Q + 0.5) / (banks * runs * occ * narrow * lanes);
                    // an item of fewer rows takes as long as a full one (one unit per thread)
                    const int items_h = (f.Hout + TH - 1) / TH;
                    const double fill_h = static_cast<double>(f.Hout) / (static_cast<double>(items_h) * TH);
                    const double t_compute = rows_per_cta / fill_h * TW * GS * f.npts * cpp / clk;
                    const double t_start = static_cast<double>(nsm) * (static_cast<double>(nrows) * rowB + rec) / 6.5e6;
                    double t_wait = 0.0;
                    if (NR < 2 * nrows) t_wait += rows_per_cta / f.Hout * (1.0 + static_cast<double>(nrows) * rowB / (100.0 * clk));
                    if (!img && NR < nrows + TH * s) t_wait += rows_per_cta / TH * 1.0;
                    const double t_depth = nrec >= 3 ? 0.0 : 0.01 * t_compute;
                    const double score = 1.0 / (t_compute + t_start + t_wait + t_depth);
                    if (score > best.score) {
                        best = RingShape{GS, R, TW, TH, nrec, NR, units, threads, slot, rec, WW, UH, UW, c2, img ? 1 : 0,
                                         smem, score, TW * GS * f.npts * cpp / clk,
                                         1.0 + static_cast<double>(nrows) * rowB / (100.0 * clk)};
                    }
                }
            }
        }
    }
    return best;
}

// The ring kernel's shape for a forward (score < 0: it does not fit): window
// kind, halo, group subset, band, item height and ring depth.
template <typename T>
RingShape choose_ring_shape(const FwdParams& f, int nsm) {
    // The halo: among target - 1 .. target + 1, the one whose best plan (at least
    // 8 consumer warps, or a whole item of a small image) has the shortest
    // estimated time, with 5 % added per pixel below target + 1 and 10 % more
    // below the target, for the samples a smaller window sends to the global
    // pass (the offsets' spread is not known here). Smaller halos only when
    // nothing in that range fits. Judged for a nominal batch of 64 whole images
    // on 148 SMs, so that it depends on the image geometry alone: an image's
    // result depends neither on N nor on the band of output rows a launch
    // covers (row0, Hout).
    const int Rt = target_halo(f.dilation);
    int Rhi = Rt + 1, Rlo = std::max(1, Rt - 1);
    const int force_halo = env_int("DCNV4_HALO", 0);
    if (force_halo > 0) Rhi = Rlo = force_halo;
    FwdParams nominal = f;
    nominal.N = 64;
    nominal.row0 = 0;
    nominal.Hout = (f.H + 2 * f.pad - f.dilation * (f.K - 1) - 1) / f.stride + 1;  // the whole image's rows
    const int min_units = std::min(256, nominal.Hout * f.Wout * f.G);
    int R = -1;
    double best_t = 0.0;
    for (int r = Rhi; r >= Rlo; --r) {
        const RingShape c = best_ring_shape<T>(nominal, r, 148, min_units);
        if (c.score <= 0.0) continue;
        const double t = (1.0 + 0.05 * (Rhi - r) + (r < Rt ? 0.1 : 0.0)) / c.score;
        if (R < 0 || t < best_t) { R = r; best_t = t; }
    }
    for (int r = Rlo - 1; r >= 1 && R < 0; --r)
        if (best_ring_shape<T>(nominal, r, 148, min_units).score > 0.0) R = r;
    // Image windows serve every offset from shared memory (a sample outside one
    // has no corner inside the image and adds nothing), so they are taken
    // whenever their estimated time is no longer than the unit windows' best,
    // judged for the same nominal batch. DCNV4_WINDOW=unit|image forces the
    // choice where it fits; a forced halo means unit windows.
    const char* wenv = std::getenv("DCNV4_WINDOW");
    const bool force_unit = force_halo > 0 || (wenv && std::strcmp(wenv, "unit") == 0);
    const bool force_img = !force_unit && wenv && std::strcmp(wenv, "image") == 0;
    bool img = false;
    if (!force_unit && image_window_fits(nominal)) {
        const RingShape c = best_ring_shape<T>(nominal, 0, 148, min_units, true);
        img = c.score > 0.0 && (force_img || R < 0 || 1.0 / c.score <= best_t);
    }
    RingShape none{};
    none.score = -1.0;
    if (R < 0 && !img) return none;
    RingShape sh = best_ring_shape<T>(f, img ? 0 : R, nsm, std::min(256, f.Hout * f.Wout * f.G), img);
    // a band of a few output rows may hold no item of 256 units in the group subsets whose
    // windows fit: then any item size, with the window kind and halo of the whole image
    if (sh.score <= 0.0 && f.Hout < nominal.Hout) sh = best_ring_shape<T>(f, img ? 0 : R, nsm, 1, img);
    return sh;
}

// choose_ring_shape costs 15-25 us of host time (a few thousand candidate
// plans); forwards of the same geometry, storage type, SM count and planner
// overrides reuse its result.
template <typename T>
RingShape cached_ring_shape(const FwdParams& f, int nsm) {
    static std::mutex mu;
    static std::map<std::string, RingShape> cache;
    char key[512];
    const char* names[] = {"DCNV4_HALO", "DCNV4_WINDOW", "DCNV4_TILE", "DCNV4_GS", "DCNV4_NREC", "DCNV4_RING"};
    int n = std::snprintf(key, sizeof key, "%d %d %d %d %d %d %d %d %d %d %d %d %d %d %d", static_cast<int>(sizeof(T)),
                          f.N, f.H, f.W, f.C, f.G, f.K, f.stride, f.pad, f.dilation, f.flags, f.npts, f.Hout, f.Wout, nsm);
    for (const char* e : names) {  // at most 46 bytes each: the key stays within its 512 bytes
        const char* v = std::getenv(e);
        if (n < 0 || n >= static_cast<int>(sizeof key)) break;
        n += std::snprintf(key + n, sizeof key - n, " %s=%.32s", e, v ? v : "");
    }
    std::lock_guard<std::mutex> lock(mu);
    if (auto it = cache.find(key); it != cache.end()) return it->second;
    const RingShape sh = choose_ring_shape<T>(f, nsm);
    if (cache.size() >= 256) cache.clear();
    cache.emplace(key, sh);
    return sh;
}

// Chooses the halo, group subset, band, item height and ring depth for the
// ring kernel and encodes the tensor map of x; false when the shape or the
// alignment does not suit it. The halo (the only choice that changes which
// samples take the window path) depends on the geometry alone, so an image's
// result never depends on the batch it comes in.
template <typename T>
bool plan_ring(const void* x, const void* om, const void* out, const FwdParams& f, unsigned* status, int4* trace,
               RingPlan* plan) {
    constexpr int E = sizeof(T);
    const int row_bytes = f.Cg * E;
    if (!aligned(x, 16) || !aligned(out, 16) || (f.C * E) % 16 || row_bytes % 16) return false;
    const int Q = row_bytes / 16;
    if (!(Q == 1 || Q == 2 || Q == 4 || Q == 5 || Q == 8)) return false;
    if (f.KK > 64) return false;  // the per-unit mask of points outside the window has 64 bits
    const int nsm = sm_count();
    if (nsm <= 0) return false;
    const RingShape sh = cached_ring_shape<T>(f, nsm);
    if (sh.score < 0.0) return false;

    dcnv4::RingParams bp{};
    bp.f = f;
    bp.TH = sh.TH; bp.TW = sh.TW; bp.GS = sh.GS; bp.nsub = f.G / sh.GS; bp.R = sh.R;
    bp.img = sh.img;
    bp.UH = sh.UH; bp.UW = sh.UW; bp.WW = sh.WW; bp.NR = sh.NR;
    bp.PB = sh.GS * row_bytes;
    bp.rowB = (sh.WW * bp.PB + 127) / 128 * 128;
    bp.cblk = sh.GS * f.Cg / sh.c2;
    bp.bands = (f.Wout + sh.TW - 1) / sh.TW;
    const long long rows_total = static_cast<long long>(f.N) * bp.bands * bp.nsub * f.Hout;
    if (rows_total >= (1LL << 31)) return false;
    bp.rows_total = static_cast<int>(rows_total);
    // Entering a strip costs a CTA its window load. When the ring cannot load the next strip's
    // window during the current strip and most CTAs enter at most two strips, the CTAs that enter
    // two run ~4 % longer (measured per CTA on the high-resolution shape): the rows are then shared
    // out by cost, each strip charging twice its estimated window-load time in rows
    // (DCNV4_STRIP_COST sets the charge for tuning runs).
    {
        const int nrows = sh.img ? sh.UH : (sh.TH - 1) * f.stride + sh.UH;
        const double rows_per_cta = static_cast<double>(rows_total) / nsm;
        int P = 0;
        if (sh.NR < 2 * nrows && rows_per_cta <= f.Hout && sh.row_us > 0.0)
            P = static_cast<int>(std::lround(2.0 * sh.strip_us / sh.row_us));
        P = env_int("DCNV4_STRIP_COST", P);
        bp.strip_cost = std::min(std::max(0, P), 1 << 16);
    }
    bp.units = sh.units;
    bp.run_slot = sh.slot;
    bp.rec_bytes = sh.rec;
    bp.ring_bytes = static_cast<int>((static_cast<size_t>(sh.NR + 1) * bp.rowB + 127) / 128 * 128);
    bp.nrec = sh.nrec;
    const size_t om_bytes = static_cast<size_t>(f.N) * f.Hout * f.Wout * f.G * 3 * f.npts * E;
    bp.om_lo = reinterpret_cast<unsigned long long>(om);
    bp.om_hi = bp.om_lo + om_bytes;
    bp.div_tw_gs = dcnv4::make_fastdiv(sh.TW * sh.GS);
    bp.div_gs = dcnv4::make_fastdiv(sh.GS);
    bp.div_nsub = dcnv4::make_fastdiv(bp.nsub);
    bp.div_bands = dcnv4::make_fastdiv(bp.bands);
    bp.div_hout = dcnv4::make_fastdiv(f.Hout);
    bp.status = status;
    bp.trace = trace;

    auto encode = tensor_map_encoder();
    if (!encode) return false;
    const int c2 = sh.c2;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(c2), static_cast<cuuint64_t>(f.C / c2),
                                static_cast<cuuint64_t>(f.W), static_cast<cuuint64_t>(f.H),
                                static_cast<cuuint64_t>(f.N)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(c2) * E, static_cast<cuuint64_t>(f.C) * E,
                                   static_cast<cuuint64_t>(f.W) * f.C * E,
                                   static_cast<cuuint64_t>(f.H) * f.W * f.C * E};
    // one ring row per load: WW pixels of GS*Cg channels
    const cuuint32_t box[5] = {static_cast<cuuint32_t>(c2), static_cast<cuuint32_t>(bp.cblk),
                               static_cast<cuuint32_t>(sh.WW), 1u, 1u};
    const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
    if (encode(&plan->map, tma_dtype<T>(), 5, const_cast<void*>(x), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    plan->p = bp;
    plan->smem = sh.smem;
    plan->threads = sh.threads;
    if (const char* d = std::getenv("DCNV4_DEBUG"); d && *d == '1')
        std::fprintf(stderr,
                     "dcnv4 ring plan: %s windows, item %dx%d GS %d (nsub %d) R %d window %dx%d width %d PB %d "
                     "ring %d rows rows_total %d units %d threads %d nrec %d smem %zu est %.1f us strip cost %d\n",
                     bp.img ? "image" : "unit", bp.TH, bp.TW, bp.GS, bp.nsub, bp.R, bp.UH, bp.UW, bp.WW, bp.PB, bp.NR,
                     bp.rows_total, bp.units, sh.threads, bp.nrec, sh.smem, 1.0 / sh.score, bp.strip_cost);
    return true;
}

// fp16 storage: weights rounded to fp16 for the mixed-precision FMA (default)
// or kept in fp32 (DCNV4_F16_EXACT=1, for comparisons).
bool f16_exact_from_env() {
    const char* v = std::getenv("DCNV4_F16_EXACT");
    return v && *v == '1';
}

template <typename T, int Q, int KS, bool HW, int PBC, bool VF, bool TRACE>
int launch_ring_q(const T* x, const T* om, T* out, const RingPlan& plan, cudaStream_t stream) {
    auto kern = dcnv4::fwd_ring_kernel<T, Q, KS, HW, PBC, VF, TRACE>;
    const cudaError_t attr = smem_limit_once(reinterpret_cast<const void*>(kern), static_cast<int>(kTileSmemLimit));
    const bool dbg = std::getenv("DCNV4_DEBUG") != nullptr;
    if (attr != cudaSuccess) {
        if (dbg) std::fprintf(stderr, "dcnv4 ring launch: shared-memory attribute: %s\n", cudaGetErrorString(attr));
        return DCNV4_ERR_LAUNCH;
    }
    // resident CTAs per SM for this block size and shared memory (looked up once per pair)
    static std::mutex occ_mu;
    static std::map<std::pair<int, size_t>, int> occ_cache;
    int per_sm = 0;
    cudaError_t occ = cudaSuccess;
    {
        std::lock_guard<std::mutex> lock(occ_mu);
        const auto key = std::make_pair(plan.threads, plan.smem);
        if (auto it = occ_cache.find(key); it != occ_cache.end()) {
            per_sm = it->second;
        } else {
            occ = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, plan.threads, plan.smem);
            if (occ == cudaSuccess && per_sm >= 1) occ_cache.emplace(key, per_sm);
        }
    }
    if (occ != cudaSuccess || per_sm < 1) {
        if (dbg) std::fprintf(stderr, "dcnv4 ring launch: occupancy %d (%s) for %d threads, %zu bytes\n", per_sm,
                              cudaGetErrorString(occ), plan.threads, plan.smem);
        return DCNV4_ERR_LAUNCH;
    }
    const long long slots = static_cast<long long>(sm_count()) * per_sm;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(plan.p.rows_total, slots));
    // programmatic stream serialisation: the CTAs may launch (and set up their
    // barriers) while the previous kernel on the stream drains; the kernel waits
    // for it before its first global access (DCNV4_PDL=0: plain serialisation)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(static_cast<unsigned>(plan.threads));
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = pdl;
    cfg.numAttrs = env_int("DCNV4_PDL", 1) != 0 ? 1 : 0;
    cudaError_t le = cudaLaunchKernelEx(&cfg, kern, plan.map, x, om, out, plan.p);
    if (le == cudaSuccess) le = cudaGetLastError();
    if (le != cudaSuccess && dbg) std::fprintf(stderr, "dcnv4 ring launch: %s\n", cudaGetErrorString(le));
    return le == cudaSuccess ? DCNV4_OK : DCNV4_ERR_LAUNCH;
}

template <typename T, int Q, bool HW, bool VF>
int launch_ring_v(const T* x, const T* om, T* out, const RingPlan& plan, cudaStream_t s) {
    // the plain forward with a 128-byte window pixel (the common case) takes the pitch as a constant
    if constexpr (!VF && Q != 5) {
        if (plan.p.PB == 128) {
            if (plan.p.f.K == 3) return launch_ring_q<T, Q, 3, HW, 128, false, false>(x, om, out, plan, s);
            return launch_ring_q<T, Q, 0, HW, 128, false, false>(x, om, out, plan, s);
        }
    }
    if (plan.p.f.K == 3) return launch_ring_q<T, Q, 3, HW, 0, VF, false>(x, om, out, plan, s);
    return launch_ring_q<T, Q, 0, HW, 0, VF, false>(x, om, out, plan, s);
}

template <typename T, int Q, bool HW>
int launch_ring_k(const T* x, const T* om, T* out, const RingPlan& plan, cudaStream_t s) {
    // the variant flags and the trace get their own instantiations, so that the
    // plain forward carries none of their code. The tracing build is the generic
    // one (runtime K and pixel pitch): those template constants change neither the
    // arithmetic nor its order, so its output is the forward's bit for bit.
    if (plan.p.trace) return launch_ring_q<T, Q, 0, HW, 0, false, true>(x, om, out, plan, s);
    if (plan.p.f.flags != 0) return launch_ring_v<T, Q, HW, true>(x, om, out, plan, s);
    return launch_ring_v<T, Q, HW, false>(x, om, out, plan, s);
}

template <typename T, int Q>
int launch_ring_k(const T* x, const T* om, T* out, const RingPlan& plan, cudaStream_t s) {
    if constexpr (std::is_same<T, __half>::value) {
        if (!f16_exact_from_env()) return launch_ring_k<T, Q, true>(x, om, out, plan, s);
    }
    return launch_ring_k<T, Q, false>(x, om, out, plan, s);
}

template <typename T>
int launch_ring(const void* x, const void* om, void* out, const RingPlan& plan, cudaStream_t s) {
    const T* xt = static_cast<const T*>(x);
    const T* omt = static_cast<const T*>(om);
    T* ot = static_cast<T*>(out);
    switch (plan.p.f.Cg * static_cast<int>(sizeof(T)) / 16) {
        case 1: return launch_ring_k<T, 1>(xt, omt, ot, plan, s);
        case 2: return launch_ring_k<T, 2>(xt, omt, ot, plan, s);
        case 4: return launch_ring_k<T, 4>(xt, omt, ot, plan, s);
        case 5: return launch_ring_k<T, 5>(xt, omt, ot, plan, s);
        default: return launch_ring_k<T, 8>(xt, omt, ot, plan, s);
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

// The forward for one storage type. With `trace` non-NULL the ring kernel's
// tracing build runs (the same arithmetic, plus one int4 per sampling point);
// returns DCNV4_NOT_TRACED when the shape takes the global-gather kernel, which
// has no tracing build.
template <typename T>
int launch_forward(const void* x, const void* om, void* out, FwdParams p, unsigned* status, int4* trace,
                   cudaStream_t stream) {
    constexpr int E = sizeof(T);
    if (variant_from_env() == Variant::Auto) {
        RingPlan plan;
        if (plan_ring<T>(x, om, out, p, status, trace, &plan)) return launch_ring<T>(x, om, out, plan, stream);
    }
    const int row_bytes = p.Cg * E;
    const bool a16 = aligned(x, 16) && aligned(out, 16) && (p.C * E) % 16 == 0;
    const bool a32 = aligned(x, 32) && aligned(out, 32) && (p.C * E) % 32 == 0;
    const size_t rec_bytes = static_cast<size_t>(3) * p.npts * E;

    int lane_bytes = 0;
    if (a16 && row_bytes % 16 == 0) {
        if (a32 && row_bytes % 32 == 0)
            lane_bytes = (E == 4 && row_bytes % 64 == 0) ? 64 : 32;
        else
            lane_bytes = 16;
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
    int rc;
    // the variant flags get their own instantiations, as in the ring kernel
    if (p.flags != 0) rc = launch_gather<T, true>(xt, omt, ot, p, lane_bytes, grid, threads, smem, stream);
    else rc = launch_gather<T, false>(xt, omt, ot, p, lane_bytes, grid, threads, smem, stream);
    if (rc == DCNV4_OK && trace) return DCNV4_NOT_TRACED;
    return rc;
}
