// Shared-memory window kernel of the DCNv4 forward aggregation (sm_100a).
//
// The scattered 2x2 corner gathers are the whole cost of the op ("DCNv4：重塑视觉模型核心",
// bqwf.cn, section 2.2: memory access dominates). Served from L1 they return a
// couple of 32-byte sectors per clock; served from shared memory with a
// bank-aware layout they return the full 128 bytes per clock. So each CTA takes
// a tile of output pixels (TH x TW) and a subset of GS channel groups, brings the
// input window its samples can reach (the tile's grid positions widened by a
// halo of R pixels; zero outside the image) and the tile's offset/mask records
// into shared memory with bulk copies (cp.async.bulk on the TMA engine, one
// instruction per contiguous row, completion counted on an mbarrier), and then
// gathers from shared memory.
//
// Thread <-> work: one thread per (pixel, group) unit, covering all Cg channels
// of the unit as Q 16-byte chunks. The window stores a pixel's GS*Cg channels
// contiguously (PB bytes, a multiple of 128 when the group subset allows), so
// chunk i of a pixel always sits on bank quad i mod 8, whatever the pixel. A
// quarter warp (8 lanes = 8 consecutive units) then reads 8 distinct bank quads
// per LDS.128 when every lane starts at a rotated chunk (rot below), so each
// 128-byte shared-memory wavefront carries 128 useful bytes.
//
// Samples whose 2x2 corners fall outside the window, or whose mask value is not
// finite, take the global-memory path of the gather kernel (same arithmetic).
#pragma once

#include "dcnv4_kernels.cuh"

namespace dcnv4 {

// Device-side status word (bit flags below), read and cleared from the host
// through dcnv4_device_status().
__device__ unsigned int g_device_status;
constexpr unsigned kStatusCopyTimeout = 1u;     // a bulk-copy wait gave up in the forward kernel
constexpr unsigned kStatusSelftestTimeout = 2u; // the self-test wait gave up (expected)

// n / d for 0 <= n < 2^31 by multiply-high and shift (Granlund & Montgomery,
// "Division by invariant integers using multiplication", 1994).
struct FastDiv {
    unsigned d, mul, shift;
};

inline FastDiv make_fastdiv(unsigned d) {
    FastDiv f{d, 0u, 0u};
    unsigned s = 0;
    while ((1ull << s) < d) ++s;
    f.shift = s;
    f.mul = static_cast<unsigned>(((1ull << 32) * ((1ull << s) - d)) / d + 1ull);
    if (d == 1) f.mul = 0u;  // q = (0 + n) >> 0
    return f;
}

__device__ __forceinline__ unsigned fdiv(unsigned n, const FastDiv& f) {
    return (__umulhi(n, f.mul) + n) >> f.shift;
}

struct WinParams {
    FwdParams f;
    int TH, TW;            // output tile
    int tiles_x, tiles_y;
    int GS, nsub;          // groups per CTA, G / GS
    int R;                 // halo in pixels around the tile's grid positions
    int WH, WW;            // window extent (pixels)
    int PB;                // bytes per window pixel: GS * Cg * sizeof(T)
    int run_slot;          // shared bytes reserved per record run
    int win_off;           // shared-memory byte offset of the window
    int units;             // TH * TW * GS
    FastDiv div_tw_gs;     // TW * GS
    FastDiv div_gs;        // GS
    FastDiv div_nsub, div_tx, div_ty;
};

// ------------------------------------------------------ mbarrier + bulk copy ---

__device__ __forceinline__ unsigned smem_addr(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Waits for phase `parity` of `bar`, giving up after `limit_ns` nanoseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, uint64_t limit_ns) {
    const uint64_t t0 = global_ns();
    for (unsigned i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && global_ns() - t0 > limit_ns) return false;
    }
}
// global -> shared bulk copy of `bytes` (multiple of 16; both addresses 16-byte
// aligned), completion counted on `bar`. No cluster multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// expect + issue one bulk copy (called by the issuing thread)
__device__ __forceinline__ void bulk_g2s_counted(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    mbar_expect_tx(bar, bytes);
    bulk_g2s(dst, src, bytes, bar);
}

constexpr uint64_t kCopyWaitLimitNs = 1000000000ull;  // 1 s

// ------------------------------------------------------------ chunk math ---

// fp32 FMA of one 16-byte chunk (16/sizeof(T) channels) into acc (pairs)
template <typename T>
__device__ __forceinline__ void fma_chunk(float2* acc, float w, const uint4& v) {
    const float2 ww = make_float2(w, w);
    if constexpr (sizeof(T) == 4) {
        acc[0] = __ffma2_rn(ww, make_float2(__uint_as_float(v.x), __uint_as_float(v.y)), acc[0]);
        acc[1] = __ffma2_rn(ww, make_float2(__uint_as_float(v.z), __uint_as_float(v.w)), acc[1]);
    } else {
        acc[0] = __ffma2_rn(ww, unpack2(v.x, static_cast<T*>(nullptr)), acc[0]);
        acc[1] = __ffma2_rn(ww, unpack2(v.y, static_cast<T*>(nullptr)), acc[1]);
        acc[2] = __ffma2_rn(ww, unpack2(v.z, static_cast<T*>(nullptr)), acc[2]);
        acc[3] = __ffma2_rn(ww, unpack2(v.w, static_cast<T*>(nullptr)), acc[3]);
    }
}

template <typename T>
__device__ __forceinline__ uint4 pack_chunk(const float2* a) {
    uint4 v;
    if constexpr (sizeof(T) == 4) {
        v.x = __float_as_uint(a[0].x); v.y = __float_as_uint(a[0].y);
        v.z = __float_as_uint(a[1].x); v.w = __float_as_uint(a[1].y);
    } else {
        v.x = pack2(a[0].x, a[0].y, static_cast<T*>(nullptr));
        v.y = pack2(a[1].x, a[1].y, static_cast<T*>(nullptr));
        v.z = pack2(a[2].x, a[2].y, static_cast<T*>(nullptr));
        v.w = pack2(a[3].x, a[3].y, static_cast<T*>(nullptr));
    }
    return v;
}

// Brings `nbytes` of global memory at `src` (aligned to the element size) to
// shared memory at slot + (src & 15): the 16-byte-aligned middle by one bulk
// copy (issued by this thread), the ragged head and tail (< 16 bytes each) by
// plain element copies. The bulk copy's byte count is posted on `bar` here.
// The caller synchronises the block before reading the slot.
template <typename T>
__device__ __forceinline__ void stage_bytes(const T* src, int count, unsigned char* slot, uint64_t* bar) {
    constexpr int E = sizeof(T);
    const uintptr_t a = reinterpret_cast<uintptr_t>(src);
    const int shift = static_cast<int>(a & 15);
    const int nbytes = count * E;
    int head = (16 - shift) & 15;
    if (head > nbytes) head = nbytes;
    const int mid = (nbytes - head) & ~15;
    const unsigned char* s = reinterpret_cast<const unsigned char*>(src);
    unsigned char* d = slot + shift;
    if (mid > 0) bulk_g2s_counted(d + head, s + head, static_cast<unsigned>(mid), bar);
    for (int i = 0; i < head / E; ++i) reinterpret_cast<T*>(d)[i] = src[i];
    for (int i = (head + mid) / E; i < count; ++i) reinterpret_cast<T*>(d)[i] = src[i];
}

// ------------------------------------------------------------ the kernel ---

template <typename T, int Q, int KS>
__global__ void __launch_bounds__(256, 2)
fwd_window_kernel(const T* __restrict__ x, const T* __restrict__ om, T* __restrict__ out, WinParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar;
    constexpr int E = sizeof(T);
    constexpr int CH = 16 / E;  // channels per 16-byte chunk
    const FwdParams& f = p.f;
    const int K = KS > 0 ? KS : f.K;
    const int KK = K * K;
    const int R3 = 3 * KK;
    const int tid = threadIdx.x;
    const int nthr = blockDim.x;

    // tile of this CTA
    const unsigned b = blockIdx.x;
    const unsigned b1 = fdiv(b, p.div_nsub);
    const int gsub = static_cast<int>(b - b1 * p.nsub);
    const unsigned b2 = fdiv(b1, p.div_tx);
    const int tx = static_cast<int>(b1 - b2 * p.tiles_x);
    const unsigned n_ = fdiv(b2, p.div_ty);
    const int ty = static_cast<int>(b2 - n_ * p.tiles_y);
    const int n = static_cast<int>(n_);
    const int ho0 = ty * p.TH, wo0 = tx * p.TW;
    const int nh = min(p.TH, f.Hout - ho0), nw = min(p.TW, f.Wout - wo0);
    const int wy0 = ho0 * f.stride - f.pad - p.R;   // window origin in image coordinates
    const int wx0 = wo0 * f.stride - f.pad - p.R;
    unsigned char* win = smem + p.win_off;
    const bool row_runs = p.GS == f.G;              // the CTA owns all groups of its pixels
    const int nruns = row_runs ? nh : nh * nw;

    if (tid == 0) mbar_init(&bar, 1);
    __syncthreads();

    // 1. window rows: the in-image part of each row arrives by bulk copy (one
    //    per row, or one per pixel when the CTA owns a subset of the groups);
    //    the rest of the window is zeroed
    const size_t pix_bytes = static_cast<size_t>(f.C) * E;
    const unsigned char* xn = reinterpret_cast<const unsigned char*>(x) +
                              static_cast<size_t>(n) * f.H * f.W * pix_bytes + static_cast<size_t>(gsub) * p.PB;
    const int xs = max(0, wx0), xe = min(f.W, wx0 + p.WW);  // in-image columns [xs, xe)
    const int ncols = xe - xs;
    if (row_runs) {
        for (int wy = tid; wy < p.WH; wy += nthr) {
            const int y = wy0 + wy;
            if (y >= 0 && y < f.H && ncols > 0)
                bulk_g2s_counted(win + (wy * p.WW + (xs - wx0)) * p.PB, xn + (static_cast<size_t>(y) * f.W + xs) * pix_bytes,
                                 static_cast<unsigned>(ncols * p.PB), &bar);
        }
    } else {
        const int npix = p.WH * max(ncols, 0);
        for (int i = tid; i < npix; i += nthr) {
            const int wy = i / ncols, c = i - (i / ncols) * ncols;
            const int y = wy0 + wy;
            if (y >= 0 && y < f.H)
                bulk_g2s_counted(win + (wy * p.WW + (xs - wx0) + c) * p.PB,
                                 xn + (static_cast<size_t>(y) * f.W + xs + c) * pix_bytes, static_cast<unsigned>(p.PB),
                                 &bar);
        }
    }
    if (wy0 < 0 || wy0 + p.WH > f.H || ncols < p.WW) {
        // zero the out-of-image part of the window (edge tiles only): whole
        // rows above/below the image, the column margins elsewhere
        const int cpp = p.PB >> 4;
        const int rowq = p.WW * cpp;
        const int left = ncols > 0 ? (xs - wx0) * cpp : rowq;
        const int right0 = ncols > 0 ? (xe - wx0) * cpp : rowq;
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int wy = 0; wy < p.WH; ++wy) {
            uint4* row = reinterpret_cast<uint4*>(win) + wy * rowq;
            const int y = wy0 + wy;
            if (y < 0 || y >= f.H) {
                for (int i = tid; i < rowq; i += nthr) row[i] = z;
            } else {
                for (int i = tid; i < left; i += nthr) row[i] = z;
                for (int i = right0 + tid; i < rowq; i += nthr) row[i] = z;
            }
        }
    }
    // 2. the tile's offset/mask records: one run per tile row when the CTA owns
    //    all groups (contiguous in memory), else one run per pixel
    for (int r = tid; r < nruns; r += nthr) {
        const int py = row_runs ? r : r / nw;
        const int px = row_runs ? 0 : r - py * nw;
        const size_t first_unit =
            (static_cast<size_t>((n * f.Hout + ho0 + py) * f.Wout + wo0 + px)) * f.G + gsub * p.GS;
        const int count = (row_runs ? nw * f.G : p.GS) * R3;
        stage_bytes<T>(om + first_unit * R3, count, smem + r * p.run_slot, &bar);
    }
    __syncthreads();                  // every expect_tx is posted
    if (tid == 0) mbar_arrive(&bar);  // the single arrival: the phase completes with the last byte
    if (!mbar_wait_bounded(&bar, 0, kCopyWaitLimitNs)) {
        atomicOr(&g_device_status, kStatusCopyTimeout);
        mbar_wait_bounded(&bar, 0, kCopyWaitLimitNs);  // let copies in flight land before leaving
        return;
    }
    __syncthreads();                  // the plain stores (zeros, record edges) too

    // 3. gather
    const int q8 = tid & 7;
    int rot = 0;
    if constexpr (Q == 2) rot = q8 >> 2;
    if constexpr (Q == 4) rot = q8 >> 1;
    if constexpr (Q == 8) rot = q8;
    const int rowB = p.WW * p.PB;
    const float wymax = static_cast<float>(p.WH - 2), wxmax = static_cast<float>(p.WW - 2);
    const int rowC = f.W * f.C;
    const T* ximg = x + static_cast<size_t>(n) * f.H * rowC;

    for (int u = tid; u < p.units; u += nthr) {
        const unsigned py_ = fdiv(static_cast<unsigned>(u), p.div_tw_gs);
        const int rem = u - static_cast<int>(py_) * p.TW * p.GS;
        const unsigned px_ = fdiv(static_cast<unsigned>(rem), p.div_gs);
        const int gl = rem - static_cast<int>(px_) * p.GS;
        const int py = static_cast<int>(py_), px = static_cast<int>(px_);
        if (py >= nh || px >= nw) continue;
        const int ho = ho0 + py, wo = wo0 + px, g = gsub * p.GS + gl;

        // this unit's record in shared memory
        const size_t first_unit =
            row_runs ? (static_cast<size_t>((n * f.Hout + ho) * f.Wout + wo0)) * f.G
                     : (static_cast<size_t>((n * f.Hout + ho) * f.Wout + wo)) * f.G + gsub * p.GS;
        const int run = row_runs ? py : py * nw + px;
        const int within = row_runs ? (px * f.G + g) : gl;
        const uintptr_t ga = reinterpret_cast<uintptr_t>(om + first_unit * R3);
        const T* rec = reinterpret_cast<const T*>(smem + run * p.run_slot + (ga & 15)) + within * R3;

        // chunk j of this thread is channel chunk (rot + j) mod Q of the unit
        int choff[Q];
#pragma unroll
        for (int j = 0; j < Q; ++j) {
            int c = rot + j;
            if (c >= Q) c -= Q;
            choff[j] = c;
        }
        const unsigned char* ubase = win + gl * (Q * 16);
        float2 acc[Q][CH / 2];
#pragma unroll
        for (int j = 0; j < Q; ++j)
#pragma unroll
            for (int i = 0; i < CH / 2; ++i) acc[j][i] = make_float2(0.f, 0.f);

        const int by = ho * f.stride - f.pad;  // grid row of ky = 0 (image coordinates)
        const int bx = wo * f.stride - f.pad;
        const float fwy = static_cast<float>(by - wy0), fwx = static_cast<float>(bx - wx0);
        const float fdil = static_cast<float>(f.dilation);

#pragma unroll (KS > 0 ? KS * KS : 1)
        for (int k = 0; k < KK; ++k) {
            const int ky = k / K, kx = k - (k / K) * K;
            const float rx = ElemTraits<T>::to_float(rec[k]);
            const float ry = ElemTraits<T>::to_float(rec[KK + k]);
            const float m = ElemTraits<T>::to_float(rec[2 * KK + k]);
            const float dy = __fmul_rn(f.offset_scale, ry);
            const float dx = __fmul_rn(f.offset_scale, rx);
            const float fy0 = floorf(dy), fx0 = floorf(dx);
            const float ly = dy - fy0, lx = dx - fx0;
            // window-relative top-left corner (exact: every term is a small integer)
            const float wyf = fy0 + (fwy + static_cast<float>(ky) * fdil);
            const float wxf = fx0 + (fwx + static_cast<float>(kx) * fdil);
            const float wy0w = 1.f - ly, wx0w = 1.f - lx;
            const float a0 = m * wy0w, a1 = m * ly;
            if (wyf >= 0.f && wyf <= wymax && wxf >= 0.f && wxf <= wxmax && fabsf(m) < INFINITY) {
                // all four corners inside the window; outside-image corners read
                // the window's zeros and the finite weight adds exactly 0
                const float w00 = a0 * wx0w, w01 = a0 * lx, w10 = a1 * wx0w, w11 = a1 * lx;
                const int off = (static_cast<int>(wyf) * p.WW + static_cast<int>(wxf)) * p.PB;
                const unsigned char* pb = ubase + off;
#pragma unroll
                for (int j = 0; j < Q; ++j) {
                    const unsigned char* pc = pb + (choff[j] << 4);
                    const uint4 v00 = *reinterpret_cast<const uint4*>(pc);
                    const uint4 v01 = *reinterpret_cast<const uint4*>(pc + p.PB);
                    const uint4 v10 = *reinterpret_cast<const uint4*>(pc + rowB);
                    const uint4 v11 = *reinterpret_cast<const uint4*>(pc + rowB + p.PB);
                    fma_chunk<T>(acc[j], w00, v00);
                    fma_chunk<T>(acc[j], w01, v01);
                    fma_chunk<T>(acc[j], w10, v10);
                    fma_chunk<T>(acc[j], w11, v11);
                }
            } else {
                // global gather with per-corner validity
                const int p0y = by + ky * f.dilation, p0x = bx + kx * f.dilation;
                const Sample s = locate(p0y, p0x, ry, rx, f.offset_scale, f.H, f.W);
                if (s.bits == 0u) continue;
                float w[4];
                w[0] = (s.bits & 1u) ? a0 * wx0w : 0.f;
                w[1] = (s.bits & 2u) ? a0 * lx : 0.f;
                w[2] = (s.bits & 4u) ? a1 * wx0w : 0.f;
                w[3] = (s.bits & 8u) ? a1 * lx : 0.f;
                const T* c00 = ximg + (s.y0 * f.W + s.x0) * f.C + g * f.Cg;
#pragma unroll
                for (int cn = 0; cn < 4; ++cn) {
                    if (!(s.bits & (1u << cn))) continue;
                    const T* pc = c00 + (cn >> 1) * rowC + (cn & 1) * f.C;
#pragma unroll
                    for (int j = 0; j < Q; ++j) {
                        uint32_t t[4];
                        load_vec<16>(pc + choff[j] * CH, t);
                        fma_chunk<T>(acc[j], w[cn], make_uint4(t[0], t[1], t[2], t[3]));
                    }
                }
            }
        }

        T* o = out + (static_cast<size_t>((n * f.Hout + ho) * f.Wout + wo)) * f.C + g * f.Cg;
#pragma unroll
        for (int j = 0; j < Q; ++j) {
            const uint4 v = pack_chunk<T>(acc[j]);
            *reinterpret_cast<uint4*>(o + choff[j] * CH) = v;
        }
    }
}

// Self-test of the bounded wait: arms an mbarrier for 16 bytes that never
// arrive (no copy is issued), waits `limit_ns`, records the timeout in the
// status word and returns. Nothing is in flight, so nothing faults or hangs.
__global__ void selftest_wait_timeout_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        mbar_expect_tx(&bar, 16);
        mbar_arrive(&bar);
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(&g_device_status, kStatusSelftestTimeout);
    }
}

}  // namespace dcnv4
