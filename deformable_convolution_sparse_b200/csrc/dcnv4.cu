// Host side of libdcnv4.so: argument checks, kernel selection and launch.
// The C ABI is declared (with the meaning of every argument) in include/dcnv4.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <cmath>
#include <mutex>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "dcnv4.h"
#include "dcnv4_kernels.cuh"
#include "dcnv4_window.cuh"
#include "dcnv4_backward.cuh"
#include "dcnv4_predictor.cuh"

namespace {

using dcnv4::FwdParams;

int elem_size(int dtype) {
    switch (dtype) {
        case DCNV4_F32: return 4;
        case DCNV4_F16: return 2;
        case DCNV4_BF16: return 2;
        default: return 0;
    }
}

bool aligned(const void* p, int a) { return (reinterpret_cast<uintptr_t>(p) % static_cast<uintptr_t>(a)) == 0; }

bool overlap(const void* a, long long abytes, const void* b, long long bbytes) {
    if (abytes <= 0 || bbytes <= 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
    return a0 < b0 + static_cast<uintptr_t>(bbytes) && b0 < a0 + static_cast<uintptr_t>(abytes);
}

constexpr long long kLimit = 1LL << 31;  // element counts stay below 2^31 (32-bit indexing)

// Shape checks shared by the forward and the index dump. Fills Hout/Wout.
int check_geometry(int N, int H, int W, int K, int stride, int pad, int dilation, int* Hout, int* Wout) {
    if (N < 0) return DCNV4_ERR_SHAPE;
    const int rc = dcnv4_output_shape(H, W, K, stride, pad, dilation, Hout, Wout);
    return rc;
}

// Checks shared by every entry point that takes the full operator signature:
// geometry, groups, dtype, offset_scale and the 32-bit element counts of x,
// out and offset_mask (returned through nx, nout, nom).
int check_sizes(int N, int H, int W, int C, int G, int K, int stride, int pad, int dilation, float offset_scale,
                int dtype, long long* nx, long long* nout, long long* nom) {
    int Hout = 0, Wout = 0;
    int rc = check_geometry(N, H, W, K, stride, pad, dilation, &Hout, &Wout);
    if (rc) return rc;
    if (C <= 0 || G <= 0) return DCNV4_ERR_SHAPE;
    if (C % G) return DCNV4_ERR_GROUPS;
    if (!elem_size(dtype)) return DCNV4_ERR_DTYPE;
    if (!std::isfinite(offset_scale)) return DCNV4_ERR_SCALE;
    *nx = static_cast<long long>(N) * H * W * C;
    *nout = static_cast<long long>(N) * Hout * Wout * C;
    *nom = static_cast<long long>(N) * Hout * Wout * G * 3 * K * K;
    if (*nx >= kLimit || *nout >= kLimit || *nom >= kLimit) return DCNV4_ERR_TOO_LARGE;
    return DCNV4_OK;
}

int launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DCNV4_OK : DCNV4_ERR_LAUNCH;
}

// ------------------------------------------------------------ dispatch ---

constexpr int kThreads = 256;

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

constexpr size_t kTileSmemLimit = 226 * 1024;  // dynamic shared memory per CTA (sm_100: 227 KB with the static part)
constexpr int kTileUnitsMax = 512;  // consumer threads (16 warps) per CTA, plus one producer warp

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

template <typename T> CUtensorMapDataType tma_dtype();
template <> CUtensorMapDataType tma_dtype<float>() { return CU_TENSOR_MAP_DATA_TYPE_FLOAT32; }
template <> CUtensorMapDataType tma_dtype<__half>() { return CU_TENSOR_MAP_DATA_TYPE_FLOAT16; }
template <> CUtensorMapDataType tma_dtype<__nv_bfloat16>() { return CU_TENSOR_MAP_DATA_TYPE_BFLOAT16; }

struct TilePlan {
    dcnv4::TileParams p;
    CUtensorMap map;
    size_t smem;
    int threads;
};

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}

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
        // bank conflicts (see the kernel); other strides pay for some
        const double banks = (PB % 128 == 0) ? 1.0 : 0.6;
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
    if (attr != cudaSuccess) return DCNV4_ERR_LAUNCH;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, plan.threads, plan.smem) != cudaSuccess || per_sm < 1)
        return DCNV4_ERR_LAUNCH;
    const long long slots = static_cast<long long>(sm_count()) * per_sm;
    const unsigned grid = static_cast<unsigned>(std::min<long long>(plan.p.tiles, slots));
    kern<<<grid, plan.threads, plan.smem, stream>>>(plan.map, x, om, out, plan.p);
    return launch_status();
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
    const bool k3 = p.K == 3;
    if (lane_bytes == 64) {
        if (k3) dcnv4::fwd_vector_kernel<T, 32, 64, 3><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 32, 64, 0><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else if (lane_bytes == 32) {
        if (k3) dcnv4::fwd_vector_kernel<T, 32, 32, 3><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 32, 32, 0><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else if (lane_bytes == 16) {
        if (k3) dcnv4::fwd_vector_kernel<T, 16, 16, 3><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_vector_kernel<T, 16, 16, 0><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    } else {
        if (k3) dcnv4::fwd_scalar_kernel<T, 3><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
        else dcnv4::fwd_scalar_kernel<T, 0><<<grid, threads, smem, stream>>>(xt, omt, ot, p);
    }
    return launch_status();
}

// Backward: grad_x is cleared on the stream, then one kernel computes every
// gradient. Vector path (4 channels per thread, float4 reductions) when the
// pointers and channel counts allow it, element path otherwise.
template <typename T>
int launch_backward(const void* x, const void* om, const void* go, float* gx, float* gom, FwdParams p,
                    cudaStream_t stream) {
    constexpr int E = sizeof(T);
    const bool vec = aligned(x, 4 * E) && aligned(go, 4 * E) && aligned(gx, 16) && p.C % 4 == 0 && p.Cg % 4 == 0;
    const int cpl = vec ? 4 : 1;
    p.chunks = p.Cg / cpl;
    int lanes = 1;
    while (lanes < p.chunks && lanes < 32) lanes <<= 1;
    p.lanes = lanes;
    // units per block: full warps, records and fp32 gradient records in shared memory
    const size_t R = static_cast<size_t>(3) * p.KK;
    const int step = lanes < 32 ? 32 / lanes : 1;
    auto smem_for = [&](int upb) {
        return ((upb * R * E + 16 + 15) & ~static_cast<size_t>(15)) + upb * R * sizeof(float);
    };
    int upb = kThreads / lanes;
    while (upb > step && smem_for(upb) > 48 * 1024) upb -= step;
    p.units_per_block = upb;
    const size_t smem = smem_for(upb);
    const long long blocks = (static_cast<long long>(p.units) + upb - 1) / upb;
    if (blocks > 0x7fffffffLL) return DCNV4_ERR_TOO_LARGE;

    const size_t gx_bytes = static_cast<size_t>(p.N) * p.H * p.W * p.C * sizeof(float);
    if (cudaMemsetAsync(gx, 0, gx_bytes, stream) != cudaSuccess) return DCNV4_ERR_CUDA;
    const T* xt = static_cast<const T*>(x);
    const T* omt = static_cast<const T*>(om);
    const T* got = static_cast<const T*>(go);
    const int threads = upb * lanes;
    auto run = [&](auto kernel) -> int {
        if (smem > 48 * 1024 &&
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
                cudaSuccess)
            return DCNV4_ERR_LAUNCH;
        kernel<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(xt, omt, got, gx, gom, p);
        return launch_status();
    };
    const bool k3 = p.K == 3;
    if (vec) return k3 ? run(dcnv4::bwd_kernel<T, 4, 3>) : run(dcnv4::bwd_kernel<T, 4, 0>);
    return k3 ? run(dcnv4::bwd_kernel<T, 1, 3>) : run(dcnv4::bwd_kernel<T, 1, 0>);
}

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
            unsigned cols = 32;
            while (cols < 2u * static_cast<unsigned>(p.NP)) cols <<= 1;
            p.tmem_cols = cols;
            p.a_fmt = std::is_same<T, __half>::value ? 0 : 1;
            const size_t b_bytes = static_cast<size_t>(p.kblocks) * p.NP * 128;
            const size_t a_stage = static_cast<size_t>(p.kblocks) * 128 * 128;
            const size_t meta = static_cast<size_t>(p.NO) * 8 + 8 + 8 * 16 + 16;
            // two output staging buffers (store of tile i overlaps the epilogue of tile i+1) when they fit
            size_t o_bytes = 0, fixed = 0;
            int stages = 0;
            for (int ob = 2; ob >= 1 && stages < 2; --ob) {
                o_bytes = (static_cast<size_t>(ob) * 128 * p.NO * E + 15) / 16 * 16;
                fixed = 1024 + b_bytes + o_bytes + meta;
                stages = 4;
                while (stages >= 2 && fixed + stages * a_stage > kTileSmemLimit) --stages;
                p.out_bufs = ob;
            }
            tc = stages >= 2;
            if (tc) {
                p.stages = stages;
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
                    auto kern = dcnv4::predictor_tc_kernel<T>;
                    static std::once_flag once;
                    static cudaError_t attr = cudaSuccess;
                    std::call_once(once, [&] {
                        attr = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                    static_cast<int>(kTileSmemLimit));
                    });
                    if (attr != cudaSuccess) return DCNV4_ERR_LAUNCH;
                    const int nsm = sm_count();
                    if (nsm <= 0) return DCNV4_ERR_CUDA;
                    const unsigned grid = static_cast<unsigned>(std::min(p.tiles, nsm));
                    if (std::getenv("DCNV4_DEBUG"))
                        std::fprintf(stderr, "dcnv4 predictor: tcgen05 NP %d kblocks %d stages %d out bufs %d tiles %d "
                                     "grid %u smem %zu tmem cols %u\n", p.NP, p.kblocks, p.stages, p.out_bufs, p.tiles,
                                     grid, smem, p.tmem_cols);
                    kern<<<grid, dcnv4::kPredThreads, smem, stream>>>(amap, bmap, bias, static_cast<T*>(rec), p);
                    return launch_status();
                }
            }
        }
    }
    // 8 warps per block, 4 pixels per warp; the pixels' inputs staged as fp32 in shared memory
    const size_t psmem = static_cast<size_t>(32) * p.C * sizeof(float);
    if (psmem > kTileSmemLimit) return DCNV4_ERR_SHAPE;
    if (psmem > 48 * 1024) {
        static std::once_flag once;
        static cudaError_t attr = cudaSuccess;
        std::call_once(once, [&] {
            attr = cudaFuncSetAttribute(dcnv4::predictor_plain_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(kTileSmemLimit));
        });
        if (attr != cudaSuccess) return DCNV4_ERR_LAUNCH;
    }
    const long long wblocks = (static_cast<long long>(p.M) + 31) / 32;
    const unsigned blocks = static_cast<unsigned>(std::min<long long>(wblocks, 148LL * 8));
    dcnv4::predictor_plain_kernel<T><<<blocks, 256, psmem, stream>>>(
        static_cast<const T*>(y), static_cast<const T*>(w), bias, static_cast<T*>(rec), p);
    return launch_status();
}

// Two non-blocking streams per device for the host-memory entry point,
// created on first use and kept for the life of the process.
constexpr int kMaxDevices = 64;
struct HostPipe {
    cudaStream_t s[2] = {nullptr, nullptr};
    bool ready = false;
};
HostPipe g_pipes[kMaxDevices];
std::mutex g_pipe_mutex;

int host_pipe(HostPipe** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DCNV4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    HostPipe& p = g_pipes[dev];
    if (!p.ready) {
        for (int i = 0; i < 2; ++i)
            if (cudaStreamCreateWithFlags(&p.s[i], cudaStreamNonBlocking) != cudaSuccess) return DCNV4_ERR_CUDA;
        p.ready = true;
    }
    *out = &p;
    return DCNV4_OK;
}

FwdParams make_params(int N, int H, int W, int C, int G, int K, int stride, int pad, int dilation,
                      float offset_scale, int Hout, int Wout, unsigned flags = 0u,
                      const void* center_logit = nullptr) {
    FwdParams p{};
    p.N = N; p.H = H; p.W = W; p.C = C; p.G = G; p.K = K; p.KK = K * K; p.Cg = C / G;
    p.stride = stride; p.pad = pad; p.dilation = dilation;
    p.Hout = Hout; p.Wout = Wout;
    p.units = N * Hout * Wout * G;
    p.offset_scale = offset_scale;
    p.flags = static_cast<int>(flags);
    const bool rc = (flags & DCNV4_FLAG_REMOVE_CENTER) != 0u;
    p.npts = p.KK - (rc ? 1 : 0);
    p.kc = rc ? (p.KK - 1) / 2 : p.KK;
    p.center_logit = center_logit;
    return p;
}

// Points per unit for a flag set (K*K, or K*K - 1 without the centre).
int points_per_unit(int K, unsigned flags) { return K * K - ((flags & DCNV4_FLAG_REMOVE_CENTER) ? 1 : 0); }

}  // namespace

extern "C" {

int dcnv4_abi_version(void) { return DCNV4_ABI_VERSION; }

const char* dcnv4_strerror(int status) {
    switch (status) {
        case DCNV4_OK: return "ok";
        case DCNV4_ERR_NULL: return "a required pointer is NULL";
        case DCNV4_ERR_SHAPE: return "invalid shape or convolution geometry";
        case DCNV4_ERR_GROUPS: return "C is not a multiple of G";
        case DCNV4_ERR_DTYPE: return "unknown dtype";
        case DCNV4_ERR_ALIGN: return "a pointer is not aligned to its element size";
        case DCNV4_ERR_ALIAS: return "an output buffer overlaps an input buffer";
        case DCNV4_ERR_SCALE: return "offset_scale is not finite";
        case DCNV4_ERR_TOO_LARGE: return "an element count reaches 2^31";
        case DCNV4_ERR_LAUNCH: return "kernel launch failed";
        case DCNV4_ERR_CUDA: return "CUDA runtime call failed";
        case DCNV4_ERR_STAGING: return "one image does not fit half of the static staging area";
        case DCNV4_ERR_FLAGS: return "unknown variant flag";
        default: return "unknown status";
    }
}

int dcnv4_output_shape(int H, int W, int K, int stride, int pad, int dilation, int* Hout, int* Wout) {
    if (H <= 0 || W <= 0 || K <= 0 || K > DCNV4_MAX_K || stride <= 0 || dilation <= 0 || pad < 0)
        return DCNV4_ERR_SHAPE;
    if (H > DCNV4_MAX_EXTENT || W > DCNV4_MAX_EXTENT || pad > DCNV4_MAX_EXTENT ||
        stride > DCNV4_MAX_EXTENT || dilation > DCNV4_MAX_EXTENT)
        return DCNV4_ERR_SHAPE;
    const long long span_h = static_cast<long long>(H) + 2LL * pad - static_cast<long long>(dilation) * (K - 1) - 1;
    const long long span_w = static_cast<long long>(W) + 2LL * pad - static_cast<long long>(dilation) * (K - 1) - 1;
    if (span_h < 0 || span_w < 0) return DCNV4_ERR_SHAPE;
    const long long ho = span_h / stride + 1, wo = span_w / stride + 1;
    // every grid coordinate p0 = o*stride - pad + k*dilation lies in [-pad, extent + pad - 1]
    if (ho > DCNV4_MAX_EXTENT || wo > DCNV4_MAX_EXTENT) return DCNV4_ERR_SHAPE;
    if (Hout) *Hout = static_cast<int>(ho);
    if (Wout) *Wout = static_cast<int>(wo);
    return DCNV4_OK;
}

int dcnv4_validate_ex(const void* x, const void* offset_mask, const void* center_logit, const void* out,
                      int N, int H, int W, int C, int G, int K,
                      int stride, int pad, int dilation, float offset_scale, int dtype, unsigned flags) {
    long long nx = 0, nout = 0, nom = 0;
    int rc = check_sizes(N, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype, &nx, &nout, &nom);
    if (rc) return rc;
    if (flags & ~static_cast<unsigned>(DCNV4_FLAG_SOFTMAX | DCNV4_FLAG_REMOVE_CENTER | DCNV4_FLAG_CENTER_SCALE))
        return DCNV4_ERR_FLAGS;
    if ((flags & DCNV4_FLAG_REMOVE_CENTER) && (K % 2 == 0 || K < 3)) return DCNV4_ERR_SHAPE;
    nom = nom / (3LL * K * K) * 3LL * points_per_unit(K, flags);
    const long long ngate = nout / C * G;
    const int e = elem_size(dtype);
    if (N == 0) return DCNV4_OK;
    const bool cs = (flags & DCNV4_FLAG_CENTER_SCALE) != 0u;
    if (!x || !offset_mask || !out || (cs && !center_logit)) return DCNV4_ERR_NULL;
    if (!aligned(x, e) || !aligned(offset_mask, e) || !aligned(out, e) || (cs && !aligned(center_logit, e)))
        return DCNV4_ERR_ALIGN;
    if (overlap(out, nout * e, x, nx * e) || overlap(out, nout * e, offset_mask, nom * e) ||
        (cs && overlap(out, nout * e, center_logit, ngate * e)))
        return DCNV4_ERR_ALIAS;
    return DCNV4_OK;
}

int dcnv4_validate(const void* x, const void* offset_mask, const void* out,
                   int N, int H, int W, int C, int G, int K,
                   int stride, int pad, int dilation, float offset_scale, int dtype) {
    return dcnv4_validate_ex(x, offset_mask, nullptr, out, N, H, W, C, G, K, stride, pad, dilation, offset_scale,
                             dtype, 0u);
}

int dcnv4_forward_ex(const void* x, const void* offset_mask, const void* center_logit, void* out,
                     int N, int H, int W, int C, int G, int K,
                     int stride, int pad, int dilation, float offset_scale, int dtype, unsigned flags,
                     void* stream) {
    const int rc = dcnv4_validate_ex(x, offset_mask, center_logit, out, N, H, W, C, G, K, stride, pad, dilation,
                                     offset_scale, dtype, flags);
    if (rc) return rc;
    if (N == 0) return DCNV4_OK;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const FwdParams p = make_params(N, H, W, C, G, K, stride, pad, dilation, offset_scale, Hout, Wout, flags,
                                    (flags & DCNV4_FLAG_CENTER_SCALE) ? center_logit : nullptr);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32: return launch_forward<float>(x, offset_mask, out, p, s);
        case DCNV4_F16: return launch_forward<__half>(x, offset_mask, out, p, s);
        default: return launch_forward<__nv_bfloat16>(x, offset_mask, out, p, s);
    }
}

int dcnv4_forward(const void* x, const void* offset_mask, void* out,
                  int N, int H, int W, int C, int G, int K,
                  int stride, int pad, int dilation, float offset_scale, int dtype,
                  void* stream) {
    return dcnv4_forward_ex(x, offset_mask, nullptr, out, N, H, W, C, G, K, stride, pad, dilation, offset_scale,
                            dtype, 0u, stream);
}

int dcnv4_backward(const void* x, const void* offset_mask, const void* grad_out,
                   float* grad_x, float* grad_offset_mask,
                   int N, int H, int W, int C, int G, int K,
                   int stride, int pad, int dilation, float offset_scale, int dtype,
                   void* stream) {
    long long nx = 0, nout = 0, nom = 0;
    int rc = check_sizes(N, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype, &nx, &nout, &nom);
    if (rc) return rc;
    if (N == 0) return DCNV4_OK;
    if (!x || !offset_mask || !grad_out || !grad_x || !grad_offset_mask) return DCNV4_ERR_NULL;
    const int e = elem_size(dtype);
    if (!aligned(x, e) || !aligned(offset_mask, e) || !aligned(grad_out, e) || !aligned(grad_x, 4) ||
        !aligned(grad_offset_mask, 4))
        return DCNV4_ERR_ALIGN;
    const void* inputs[3] = {x, offset_mask, grad_out};
    const long long in_bytes[3] = {nx * e, nom * e, nout * e};
    for (int i = 0; i < 3; ++i)
        if (overlap(grad_x, nx * 4, inputs[i], in_bytes[i]) || overlap(grad_offset_mask, nom * 4, inputs[i], in_bytes[i]))
            return DCNV4_ERR_ALIAS;
    if (overlap(grad_x, nx * 4, grad_offset_mask, nom * 4)) return DCNV4_ERR_ALIAS;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const FwdParams p = make_params(N, H, W, C, G, K, stride, pad, dilation, offset_scale, Hout, Wout);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32: return launch_backward<float>(x, offset_mask, grad_out, grad_x, grad_offset_mask, p, s);
        case DCNV4_F16: return launch_backward<__half>(x, offset_mask, grad_out, grad_x, grad_offset_mask, p, s);
        default: return launch_backward<__nv_bfloat16>(x, offset_mask, grad_out, grad_x, grad_offset_mask, p, s);
    }
}

int dcnv4_predictor(const void* y, const void* weight, const float* bias, void* offset_mask,
                    int M, int C, int G, int K, unsigned flags, int dtype, void* stream) {
    if (M < 0 || C <= 0 || G <= 0 || K <= 0 || K > DCNV4_MAX_K) return DCNV4_ERR_SHAPE;
    if (flags & ~static_cast<unsigned>(DCNV4_FLAG_REMOVE_CENTER)) return DCNV4_ERR_FLAGS;
    if ((flags & DCNV4_FLAG_REMOVE_CENTER) && (K % 2 == 0 || K < 3)) return DCNV4_ERR_SHAPE;
    const int e = elem_size(dtype);
    if (!e) return DCNV4_ERR_DTYPE;
    const long long P = points_per_unit(K, flags);
    const long long NO = 3LL * G * P;
    const long long ny = static_cast<long long>(M) * C, nw = NO * C, nrec = static_cast<long long>(M) * NO;
    if (ny >= kLimit || nw >= kLimit || nrec >= kLimit) return DCNV4_ERR_TOO_LARGE;
    if (M == 0) return DCNV4_OK;
    if (!y || !weight || !offset_mask) return DCNV4_ERR_NULL;
    if (!aligned(y, e) || !aligned(weight, e) || !aligned(offset_mask, e) || (bias && !aligned(bias, 4)))
        return DCNV4_ERR_ALIGN;
    if (overlap(offset_mask, nrec * e, y, ny * e) || overlap(offset_mask, nrec * e, weight, nw * e) ||
        (bias && overlap(offset_mask, nrec * e, bias, NO * 4)))
        return DCNV4_ERR_ALIAS;
    dcnv4::PredParams p{};
    p.M = M; p.C = C; p.G = G; p.P = static_cast<int>(P); p.NO = static_cast<int>(NO);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32: return launch_predictor<float>(y, weight, bias, offset_mask, p, s);
        case DCNV4_F16: return launch_predictor<__half>(y, weight, bias, offset_mask, p, s);
        default: return launch_predictor<__nv_bfloat16>(y, weight, bias, offset_mask, p, s);
    }
}

int dcnv4_forward_host(const void* x_host, const void* offset_mask_host, void* out_host,
                       void* x_dev, void* offset_mask_dev, void* out_dev,
                       int N, int H, int W, int C, int G, int K,
                       int stride, int pad, int dilation, float offset_scale, int dtype,
                       void* stream) {
    int rc = dcnv4_validate(x_dev, offset_mask_dev, out_dev, N, H, W, C, G, K, stride, pad, dilation,
                            offset_scale, dtype);
    if (rc) return rc;
    if (N == 0) return DCNV4_OK;
    if (!x_host || !offset_mask_host || !out_host) return DCNV4_ERR_NULL;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const size_t e = static_cast<size_t>(elem_size(dtype));
    const size_t x_img = static_cast<size_t>(H) * W * C * e;
    const size_t om_img = static_cast<size_t>(Hout) * Wout * G * 3 * K * K * e;
    const size_t out_img = static_cast<size_t>(Hout) * Wout * C * e;
    if (overlap(out_host, static_cast<long long>(out_img * N), x_host, static_cast<long long>(x_img * N)) ||
        overlap(out_host, static_cast<long long>(out_img * N), offset_mask_host, static_cast<long long>(om_img * N)))
        return DCNV4_ERR_ALIAS;

    HostPipe* pipe = nullptr;
    rc = host_pipe(&pipe);
    if (rc) return rc;
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev_start = nullptr, ev_done[2] = {nullptr, nullptr};
    auto fail = [&](int code) {
        if (ev_start) cudaEventDestroy(ev_start);
        for (auto& ev : ev_done)
            if (ev) cudaEventDestroy(ev);
        return code;
    };
    if (cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming) != cudaSuccess) return fail(DCNV4_ERR_CUDA);
    for (auto& ev : ev_done)
        if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return fail(DCNV4_ERR_CUDA);
    if (cudaEventRecord(ev_start, user) != cudaSuccess) return fail(DCNV4_ERR_CUDA);
    for (int i = 0; i < 2; ++i)
        if (cudaStreamWaitEvent(pipe->s[i], ev_start, 0) != cudaSuccess) return fail(DCNV4_ERR_CUDA);

    // chunks of whole images: enough of them for the two copy directions to overlap
    const int chunks = N < 8 ? N : 8;
    const char* xh = static_cast<const char*>(x_host);
    const char* omh = static_cast<const char*>(offset_mask_host);
    char* oh = static_cast<char*>(out_host);
    char* xd = static_cast<char*>(x_dev);
    char* omd = static_cast<char*>(offset_mask_dev);
    char* od = static_cast<char*>(out_dev);
    int n0 = 0;
    for (int c = 0; c < chunks; ++c) {
        const int n1 = static_cast<int>((static_cast<long long>(N) * (c + 1)) / chunks);
        const int nc = n1 - n0;
        if (nc == 0) continue;
        cudaStream_t s = pipe->s[c & 1];
        if (cudaMemcpyAsync(xd + n0 * x_img, xh + n0 * x_img, nc * x_img, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(omd + n0 * om_img, omh + n0 * om_img, nc * om_img, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
        rc = dcnv4_forward(xd + n0 * x_img, omd + n0 * om_img, od + n0 * out_img, nc, H, W, C, G, K, stride, pad,
                           dilation, offset_scale, dtype, s);
        if (rc) return fail(rc);
        if (cudaMemcpyAsync(oh + n0 * out_img, od + n0 * out_img, nc * out_img, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
        n0 = n1;
    }
    for (int i = 0; i < 2; ++i) {
        if (cudaEventRecord(ev_done[i], pipe->s[i]) != cudaSuccess || cudaStreamWaitEvent(user, ev_done[i], 0) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
    }
    // events may be destroyed while pending: the waits already queued keep their meaning
    fail(DCNV4_OK);
    return DCNV4_OK;
}

int dcnv4_device_status(unsigned int* status, int clear) {
    if (!status) return DCNV4_ERR_NULL;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, dcnv4::g_device_status, sizeof(v)) != cudaSuccess) return DCNV4_ERR_CUDA;
    *status = v;
    if (clear) {
        const unsigned z = 0;
        if (cudaMemcpyToSymbol(dcnv4::g_device_status, &z, sizeof(z)) != cudaSuccess) return DCNV4_ERR_CUDA;
    }
    return DCNV4_OK;
}

int dcnv4_selftest_wait_timeout(unsigned long long limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > 2000000000ull) return DCNV4_ERR_SHAPE;
    dcnv4::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    return launch_status();
}

int dcnv4_sampling_index(const void* offset_mask, int32_t* corner, uint8_t* valid,
                         int N, int H, int W, int G, int K,
                         int stride, int pad, int dilation, float offset_scale, int dtype,
                         void* stream) {
    int Hout = 0, Wout = 0;
    int rc = check_geometry(N, H, W, K, stride, pad, dilation, &Hout, &Wout);
    if (rc) return rc;
    if (G <= 0) return DCNV4_ERR_SHAPE;
    const int e = elem_size(dtype);
    if (!e) return DCNV4_ERR_DTYPE;
    if (!std::isfinite(offset_scale)) return DCNV4_ERR_SCALE;
    const long long npts = static_cast<long long>(N) * Hout * Wout * G * K * K;
    if (3 * npts >= kLimit) return DCNV4_ERR_TOO_LARGE;
    if (N == 0) return DCNV4_OK;
    if (!offset_mask || !corner || !valid) return DCNV4_ERR_NULL;
    if (!aligned(offset_mask, e) || !aligned(corner, 4)) return DCNV4_ERR_ALIGN;
    if (overlap(corner, 8 * npts, offset_mask, 3 * npts * e) || overlap(valid, npts, offset_mask, 3 * npts * e) ||
        overlap(valid, npts, corner, 8 * npts))
        return DCNV4_ERR_ALIAS;
    FwdParams p = make_params(N, H, W, G, G, K, stride, pad, dilation, offset_scale, Hout, Wout);
    const long long want = (npts + 255) / 256;
    const unsigned blocks = static_cast<unsigned>(want < 148 * 32 ? want : 148 * 32);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32:
            dcnv4::sampling_index_kernel<float><<<blocks, 256, 0, s>>>(
                static_cast<const float*>(offset_mask), corner, valid, p);
            break;
        case DCNV4_F16:
            dcnv4::sampling_index_kernel<__half><<<blocks, 256, 0, s>>>(
                static_cast<const __half*>(offset_mask), corner, valid, p);
            break;
        default:
            dcnv4::sampling_index_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(offset_mask), corner, valid, p);
            break;
    }
    return launch_status();
}

}  // extern "C"

// --------------------------------------------------------------------------
// Allocation-free host entry point: staging in a fixed device array.

namespace {

__device__ __align__(256) unsigned char g_noalloc_staging[DCNV4_NOALLOC_STAGING_BYTES];

unsigned char* g_noalloc_addr[kMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the staging array on the current device, looked up once
// per device (cudaGetSymbolAddress with that device current).
int noalloc_staging(unsigned char** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DCNV4_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_staging) != cudaSuccess || !p) return DCNV4_ERR_CUDA;
        g_noalloc_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_noalloc_addr[dev];
    return DCNV4_OK;
}

size_t round256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

extern "C" int dcnv4_forward_host_noalloc(const void* x_host, const void* offset_mask_host, void* out_host,
                                          int N, int H, int W, int C, int G, int K,
                                          int stride, int pad, int dilation, float offset_scale, int dtype,
                                          void* stream) {
    // the host buffers get the checks the device buffers get elsewhere
    int rc = dcnv4_validate(x_host, offset_mask_host, out_host, N, H, W, C, G, K, stride, pad, dilation,
                            offset_scale, dtype);
    if (rc) return rc;
    if (N == 0) return DCNV4_OK;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const size_t e = static_cast<size_t>(elem_size(dtype));
    const size_t x_img = static_cast<size_t>(H) * W * C * e;
    const size_t om_img = static_cast<size_t>(Hout) * Wout * G * 3 * K * K * e;
    const size_t out_img = static_cast<size_t>(Hout) * Wout * C * e;
    const size_t half = DCNV4_NOALLOC_STAGING_BYTES / 2;
    // images per chunk: x, offset_mask and out of the chunk, each 256-byte aligned, in one half
    int per_chunk = 0;
    while (per_chunk < N && round256((per_chunk + 1) * x_img) + round256((per_chunk + 1) * om_img) +
                                    round256((per_chunk + 1) * out_img) <= half)
        ++per_chunk;
    if (per_chunk == 0) return DCNV4_ERR_STAGING;

    unsigned char* staging = nullptr;
    rc = noalloc_staging(&staging);
    if (rc) return rc;
    HostPipe* pipe = nullptr;
    rc = host_pipe(&pipe);
    if (rc) return rc;
    cudaStream_t user = static_cast<cudaStream_t>(stream);
    cudaEvent_t ev_start = nullptr, ev_done[2] = {nullptr, nullptr};
    auto release = [&](int code) {
        if (ev_start) cudaEventDestroy(ev_start);
        for (auto& ev : ev_done)
            if (ev) cudaEventDestroy(ev);
        return code;
    };
    if (cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming) != cudaSuccess) return release(DCNV4_ERR_CUDA);
    for (auto& ev : ev_done)
        if (cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return release(DCNV4_ERR_CUDA);
    if (cudaEventRecord(ev_start, user) != cudaSuccess) return release(DCNV4_ERR_CUDA);
    for (int i = 0; i < 2; ++i)
        if (cudaStreamWaitEvent(pipe->s[i], ev_start, 0) != cudaSuccess) return release(DCNV4_ERR_CUDA);

    const char* xh = static_cast<const char*>(x_host);
    const char* omh = static_cast<const char*>(offset_mask_host);
    char* oh = static_cast<char*>(out_host);
    int c = 0;
    for (int n0 = 0; n0 < N; n0 += per_chunk, ++c) {
        const int nc = std::min(per_chunk, N - n0);
        // chunk c uses half c & 1 on stream c & 1: a half is reused only by a
        // later chunk of the same stream, after this chunk's copies are done
        unsigned char* xd = staging + (c & 1) * half;
        unsigned char* omd = xd + round256(nc * x_img);
        unsigned char* od = omd + round256(nc * om_img);
        cudaStream_t s = pipe->s[c & 1];
        if (cudaMemcpyAsync(xd, xh + n0 * x_img, nc * x_img, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(omd, omh + n0 * om_img, nc * om_img, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return release(DCNV4_ERR_CUDA);
        rc = dcnv4_forward(xd, omd, od, nc, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype, s);
        if (rc) return release(rc);
        if (cudaMemcpyAsync(oh + n0 * out_img, od, nc * out_img, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return release(DCNV4_ERR_CUDA);
    }
    for (int i = 0; i < 2; ++i) {
        if (cudaEventRecord(ev_done[i], pipe->s[i]) != cudaSuccess || cudaStreamWaitEvent(user, ev_done[i], 0) != cudaSuccess)
            return release(DCNV4_ERR_CUDA);
    }
    return release(DCNV4_OK);
}
