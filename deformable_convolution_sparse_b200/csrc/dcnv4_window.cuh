// Persistent shared-memory window kernel of the DCNv4 forward aggregation (sm_100a).
//
// The scattered 2x2 corner gathers are the whole cost of the op ("DCNv4：重塑视觉模型核心",
// bqwf.cn, section 2.2: memory access dominates). Served from L1 they return a
// couple of 32-byte sectors per clock; served from shared memory with a
// bank-aware layout they return the full 128 bytes per clock. So the kernel
// works tile by tile: a tile is TH x TW output pixels of one image and a subset
// of GS channel groups. For each tile the CTA brings into shared memory
//  - the input window its samples can reach: the tile's grid positions widened
//    by a halo of R pixels, all GS*Cg channels of each pixel, as ONE TMA tensor
//    load (cp.async.bulk.tensor, 5-D map over x); pixels outside the image
//    arrive as zeros from the TMA unit itself;
//  - the tile's offset/mask records, as one bulk copy (cp.async.bulk) per
//    contiguous run (a tile row when the CTA owns all groups, else a pixel);
// both counted on one mbarrier per buffer. CTAs are persistent and double
// buffered: while the threads gather tile i from one buffer, warp 0 has
// already issued the copies of tile i+1 into the other.
//
// Thread <-> work: one thread per (pixel, group) unit, covering all Cg channels
// of the unit as Q 16-byte chunks. The window stores a pixel's GS*Cg channels
// contiguously (PB bytes, a multiple of 128 when the group subset allows), so
// chunk i of a pixel always sits on bank quad i mod 8, whatever the pixel. A
// quarter warp (8 lanes = 8 consecutive units) then reads 8 distinct bank quads
// per LDS.128 when every lane starts at a rotated chunk (rot below), so each
// 128-byte shared-memory wavefront carries 128 useful bytes.
//
// Samples whose 2x2 corners fall outside the window (offsets beyond the halo),
// or whose mask value is not finite, are marked during the pass over the
// window and gathered afterwards from global memory with per-corner validity,
// so a warp waits for that memory latency once rather than once per point.
#pragma once

#include <cuda.h>

#include "dcnv4_kernels.cuh"

namespace dcnv4 {

// Device-side status word (bit flags below), read and cleared from the host
// through dcnv4_device_status().
__device__ unsigned int g_device_status;
constexpr unsigned kStatusCopyTimeout = 1u;     // a copy wait gave up in the forward kernel
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

struct TileParams {
    FwdParams f;
    int TH, TW;             // output tile
    int tiles_x, tiles_y;
    int GS, nsub;           // groups per tile, G / GS
    int R;                  // halo in pixels around the tile's grid positions
    int WH, WW;             // window extent (pixels)
    int PB;                 // bytes per window pixel: GS * Cg * sizeof(T)
    int cblk;               // channel blocks of the tensor map per group subset
    int tiles;              // N * tiles_y * tiles_x * nsub
    int items;              // work items of the persistent loop: main_tiles + (tiles - main_tiles) * tail_split
    int main_tiles;         // tiles processed whole; the rest (the last partial wave) are split by warps
    int tail_split;         // CTAs sharing one tail tile (its consumer warps divided among them); 1: no split
    int units;              // TH * TW * GS
    int run_slot;           // shared bytes per record run
    int rec_bytes;          // one record buffer (multiple of 128)
    int win_bytes;          // one window buffer (multiple of 128)
    int nrec;               // record buffers (2 or 3); windows always use 2
    unsigned long long om_lo, om_hi;  // byte range of the offset_mask tensor
    FastDiv div_tw_gs, div_gs, div_nsub, div_tx, div_ty;
};

// ------------------------------------------------------ mbarrier + bulk copy ---

__device__ __forceinline__ unsigned smem_addr(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
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
// aligned) with its byte count posted on `bar` first. No cluster multicast.
__device__ __forceinline__ void bulk_g2s_counted(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    mbar_expect_tx(bar, bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// One TMA tile load from a 5-D tensor map (no multicast); out-of-range
// elements are written as zeros. The caller posts the byte count.
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3, int c4,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar))
        : "memory");
}

constexpr uint64_t kCopyWaitLimitNs = 1000000000ull;  // 1 s

// ------------------------------------------------------------ chunk math ---

// Accumulates w * x over one 16-byte chunk (16/sizeof(T) channels) into acc
// (pairs of fp32 accumulators).
//  - HW (fp16 storage only): the weight is rounded once to fp16 and each
//    fp16 x fp16 product, exact in fp32, is added to the fp32 accumulator by
//    one mixed-precision FMA (fma.rn.f32.f16): no conversion of x and no
//    register pairing, which halves the FMA-pipe work per channel.
//  - otherwise: x is widened to fp32 and multiplied by the fp32 weight with
//    packed fp32x2 FMAs.
template <typename T, bool HW = false>
__device__ __forceinline__ void fma_chunk(float2* acc, float w, const uint4& v) {
    if constexpr (HW && std::is_same<T, __half>::value) {
        const unsigned short wh = __half_as_ushort(__float2half_rn(w));
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            asm("{\n\t.reg .f16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
                "fma.rn.f32.f16 %0, lo, %3, %0;\n\tfma.rn.f32.f16 %1, hi, %3, %1;\n\t}"
                : "+f"(acc[q].x), "+f"(acc[q].y)
                : "r"(vw[q]), "h"(wh));
        return;
    }
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

// acc = (1 - s) * acc + s * x over one 16-byte chunk (centre feature scaling)
template <typename T>
__device__ __forceinline__ void blend_chunk(float2* acc, float s, const uint4& v) {
    const float r = 1.f - s;
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            acc[q].x = fmaf(s, __uint_as_float(vw[2 * q]), r * acc[q].x);
            acc[q].y = fmaf(s, __uint_as_float(vw[2 * q + 1]), r * acc[q].y);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 f = unpack2(vw[q], static_cast<T*>(nullptr));
            acc[q].x = fmaf(s, f.x, r * acc[q].x);
            acc[q].y = fmaf(s, f.y, r * acc[q].y);
        }
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

// ------------------------------------------------------------ tiles ---

struct TileCoord {
    int n, gsub, ho0, wo0, nh, nw, wy0, wx0;
};

__device__ __forceinline__ TileCoord tile_coord(const TileParams& p, unsigned t) {
    TileCoord c;
    const unsigned t1 = fdiv(t, p.div_nsub);
    c.gsub = static_cast<int>(t - t1 * p.nsub);
    const unsigned t2 = fdiv(t1, p.div_tx);
    const int tx = static_cast<int>(t1 - t2 * p.tiles_x);
    const unsigned n = fdiv(t2, p.div_ty);
    const int ty = static_cast<int>(t2 - n * p.tiles_y);
    c.n = static_cast<int>(n);
    c.ho0 = ty * p.TH;
    c.wo0 = tx * p.TW;
    c.nh = min(p.TH, p.f.Hout - c.ho0);
    c.nw = min(p.TW, p.f.Wout - c.wo0);
    c.wy0 = c.ho0 * p.f.stride - p.f.pad - p.R;
    c.wx0 = c.wo0 * p.f.stride - p.f.pad - p.R;
    return c;
}

// Tile of work item w of the persistent loop, and which warp slice of it the
// item covers (-1: the whole tile). The last partial wave of tiles is split
// by consumer warps over tail_split CTAs, so that it takes a fraction of a
// tile's time instead of a whole one while most SMs idle.
__device__ __forceinline__ unsigned item_tile(const TileParams& p, int w, int* part) {
    if (w < p.main_tiles) {
        *part = -1;
        return static_cast<unsigned>(w);
    }
    const int q = w - p.main_tiles;
    *part = q % p.tail_split;
    return static_cast<unsigned>(p.main_tiles + q / p.tail_split);
}

// Address and element count of record run r of a tile.
template <typename T>
__device__ __forceinline__ const unsigned char* run_src(const TileParams& p, const TileCoord& c, const T* om, int r,
                                                        int* count) {
    const FwdParams& f = p.f;
    const bool row_runs = p.GS == f.G;
    const int py = row_runs ? r : r / c.nw;
    const int px = row_runs ? 0 : r - py * c.nw;
    const size_t first_unit = (static_cast<size_t>((c.n * f.Hout + c.ho0 + py) * f.Wout + c.wo0 + px)) * f.G +
                              static_cast<size_t>(c.gsub) * p.GS;
    *count = (row_runs ? c.nw * f.G : p.GS) * 3 * f.npts;
    return reinterpret_cast<const unsigned char*>(om + first_unit * 3 * f.npts);
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc) : "memory");
}
// one arrival on `bar` once every cp.async this thread issued before has landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Arrivals the records' "full" barrier waits for: the producer's lane 0, plus
// every producer lane's cp.async arrival when the records are per pixel.
__host__ __device__ __forceinline__ unsigned rec_full_arrivals(bool row_runs) { return row_runs ? 1u : 33u; }

// Producer warp: queues the copies of tile t's offset/mask records into `buf`
// on `bar`. Runs are widened to 16-byte boundaries when that stays inside the
// offset_mask tensor (else the aligned middle is copied and the ragged ends by
// plain stores). A tile row's records are one run and go by one bulk copy
// (cp.async.bulk). When the CTA owns only some of the groups the runs are per
// pixel and short; those go by 16-byte cp.async from all 32 lanes (a bulk copy
// costs the TMA unit tens of cycles each, too many for 100+ runs).
template <typename T>
__device__ __forceinline__ void issue_records(const TileParams& p, const T* om, const TileCoord& c,
                                              unsigned char* buf, uint64_t* bar, int lane) {
    constexpr int E = sizeof(T);
    const bool row_runs = p.GS == p.f.G;
    const int nruns = row_runs ? c.nh : c.nh * c.nw;
    for (int r = lane; r < nruns; r += 32) {
        int count;
        const unsigned char* s = run_src<T>(p, c, om, r, &count);
        const unsigned long long a = reinterpret_cast<unsigned long long>(s);
        const unsigned long long b = a + static_cast<unsigned long long>(count) * E;
        unsigned long long a16 = a & ~15ull, b16 = (b + 15) & ~15ull;
        unsigned char* slot = buf + r * p.run_slot;  // byte a lands at slot + (a & 15)
        if (!(a16 >= p.om_lo && b16 <= p.om_hi)) {
            // the ragged ends by plain copies, the aligned middle below
            const unsigned long long ma = (a + 15) & ~15ull, mb = b & ~15ull;
            const T* src = reinterpret_cast<const T*>(s);
            T* dst = reinterpret_cast<T*>(slot + (a & 15));
            const int head = mb > ma ? static_cast<int>((ma - a) / E) : count;
            for (int i = 0; i < head; ++i) dst[i] = src[i];
            if (mb > ma)
                for (int i = static_cast<int>((mb - a) / E); i < count; ++i) dst[i] = src[i];
            a16 = ma;
            b16 = mb > ma ? mb : ma;
        }
        if (b16 <= a16) continue;
        unsigned char* d = slot + (a16 - (a & ~15ull));
        if (row_runs) {
            bulk_g2s_counted(d, reinterpret_cast<const void*>(a16), static_cast<unsigned>(b16 - a16), bar);
        } else {
            for (unsigned long long q = a16; q < b16; q += 16) cp_async16(d + (q - a16), reinterpret_cast<const void*>(q));
        }
    }
    if (!row_runs) cp_async_arrive_noinc(bar);
    __syncwarp();
    if (lane == 0) mbar_arrive(bar);
}

// Producer warp, lane 0: the window of tile t as one TMA load on `bar`.
__device__ __forceinline__ void issue_window(const TileParams& p, const CUtensorMap* xmap, const TileCoord& c,
                                             unsigned char* buf, uint64_t* bar, int lane) {
    if (lane == 0) {
        mbar_expect_tx(bar, static_cast<unsigned>(p.WH * p.WW * p.PB));
        tma_load_5d(buf, xmap, 0, c.gsub * p.cblk, c.wx0, c.wy0, c.n, bar);
        mbar_arrive(bar);
    }
}

// Two fp32 weights to a pair of fp16 (round to nearest even), one instruction.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// acc += w * x over one fp16 chunk with mixed-precision FMAs; `w2` holds the
// fp16 weight in its low (hi == false) or high half.
template <bool HI>
__device__ __forceinline__ void fma_chunk_h(float2* acc, uint32_t w2, const uint4& v) {
    const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if constexpr (HI)
            asm("{\n\t.reg .f16 lo, hi, wl, wh;\n\tmov.b32 {lo, hi}, %2;\n\tmov.b32 {wl, wh}, %3;\n\t"
                "fma.rn.f32.f16 %0, lo, wh, %0;\n\tfma.rn.f32.f16 %1, hi, wh, %1;\n\t}"
                : "+f"(acc[q].x), "+f"(acc[q].y)
                : "r"(vw[q]), "r"(w2));
        else
            asm("{\n\t.reg .f16 lo, hi, wl, wh;\n\tmov.b32 {lo, hi}, %2;\n\tmov.b32 {wl, wh}, %3;\n\t"
                "fma.rn.f32.f16 %0, lo, wl, %0;\n\tfma.rn.f32.f16 %1, hi, wl, %1;\n\t}"
                : "+f"(acc[q].x), "+f"(acc[q].y)
                : "r"(vw[q]), "r"(w2));
    }
}

// ------------------------------------------------------------ the kernel ---

// Warp roles: warps 0 .. nc-1 consume (gather), warp nc produces (issues the
// copies). Windows use a ring of 2 buffers, records a ring of p.nrec (2 or 3):
// records come from DRAM on first touch and get the longer lead. Every buffer
// has a "full" barrier (producer arrivals plus the copied bytes) and an
// "empty" barrier (one arrival per consumer warp once it is done with the
// tile). No CTA-wide barrier is taken after the set-up, so a warp held up by a
// global-memory gather does not stall the others. Every wait is bounded; a
// wait that gives up sets the device status word and the warp leaves (the
// producer after letting its copies in flight land).
//
// PBC: the window's pixel stride as a compile-time constant (0: p.PB).
// VF: the variant flags of p.f may be set (softmax over the masks, centre
// point removed, centre feature scaling); false compiles them out.
// Registers: capped at 112 per thread; the compiler's own choice under a
// launch bound was 96, and the extra registers keep more corner loads in
// flight. The planner keeps CTAs at 16 warps or fewer, so that each SM
// sub-partition (16 K registers) holds its share of 4 warps.
template <typename T, int Q, int KS, bool HW, int PBC, bool VF>
__global__ void __maxnreg__(112)
fwd_tile_kernel(const __grid_constant__ CUtensorMap xmap, const T* __restrict__ x, const T* __restrict__ om,
                T* __restrict__ out, TileParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t win_full[2], win_empty[2], rec_full[3], rec_empty[3];
    constexpr int E = sizeof(T);
    constexpr int CH = 16 / E;  // channels per 16-byte chunk
    const FwdParams& f = p.f;
    const int K = KS > 0 ? KS : f.K;
    const int KK = K * K;
    const int NP = VF ? f.npts : KK;   // points per unit
    const int kcs = VF ? f.kc : KK;    // grid index left out (none: KK)
    const int R3 = 3 * NP;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nc = static_cast<int>(blockDim.x >> 5) - 1;  // consumer warps
    const bool row_runs = p.GS == f.G;
    const int nrec = p.nrec;
    const int PB = PBC ? PBC : p.PB;
    unsigned char* const winbuf = smem;                          // 2 windows
    unsigned char* const recbuf = smem + 2 * p.win_bytes;        // nrec record sets

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&win_full[b], 1);
            mbar_init(&win_empty[b], static_cast<unsigned>(nc));
        }
        for (int b = 0; b < 3; ++b) {
            mbar_init(&rec_full[b], rec_full_arrivals(row_runs));
            mbar_init(&rec_empty[b], static_cast<unsigned>(nc));
        }
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    }
    __syncthreads();
    const int first = static_cast<int>(blockIdx.x);
    if (first >= p.items) return;
    const int stride_t = static_cast<int>(gridDim.x);
    const int ntiles = (p.items - first + stride_t - 1) / stride_t;  // work items of this CTA

    if (warp == nc) {
        // ---------------------------------------------------------------- producer
        // step i: the records of tile i and the window of tile i - (nrec - 2), each
        // once the consumers are done with the buffer it reuses
        const int lead = nrec - 2;
        for (int i = 0; i < ntiles + lead; ++i) {
            bool ok = true;
            if (i < ntiles && i >= nrec)
                ok = mbar_wait_bounded(&rec_empty[i % nrec], ((i / nrec) - 1) & 1, kCopyWaitLimitNs);
            const int j = i - lead;
            if (ok && j >= 2 && j < ntiles)
                ok = mbar_wait_bounded(&win_empty[j & 1], ((j >> 1) - 1) & 1, kCopyWaitLimitNs);
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicOr(&g_device_status, kStatusCopyTimeout);
                // let the copies already queued land before leaving
                for (int q = max(0, i - nrec); q < min(i, ntiles); ++q)
                    mbar_wait_bounded(&rec_full[q % nrec], (q / nrec) & 1, kCopyWaitLimitNs);
                for (int q = max(0, j - 2); q < min(j, ntiles); ++q)
                    mbar_wait_bounded(&win_full[q & 1], (q >> 1) & 1, kCopyWaitLimitNs);
                return;
            }
            fence_proxy_async();  // the consumers' reads of those buffers before the async writes
            int part_unused;
            if (i < ntiles)
                issue_records<T>(p, om, tile_coord(p, item_tile(p, first + i * stride_t, &part_unused)),
                                 recbuf + (i % nrec) * p.rec_bytes, &rec_full[i % nrec], lane);
            if (j >= 0 && j < ntiles)
                issue_window(p, &xmap, tile_coord(p, item_tile(p, first + j * stride_t, &part_unused)),
                             winbuf + (j & 1) * p.win_bytes, &win_full[j & 1], lane);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    // this thread's unit (the same in every tile) and its chunk rotation
    const int u = warp * 32 + lane;
    const bool has_unit = u < p.units;
    const int py = static_cast<int>(fdiv(static_cast<unsigned>(u), p.div_tw_gs));
    const int rem = u - py * p.TW * p.GS;
    const int px = static_cast<int>(fdiv(static_cast<unsigned>(rem), p.div_gs));
    const int gl = rem - px * p.GS;
    const int q8 = lane & 7;
    int rot = 0;
    if constexpr (Q == 2) rot = q8 >> 2;
    if constexpr (Q == 4) rot = q8 >> 1;
    if constexpr (Q == 8) rot = q8;
    int choff[Q];
#pragma unroll
    for (int j = 0; j < Q; ++j) {
        int cc = rot + j;
        if (cc >= Q) cc -= Q;
        choff[j] = cc;
    }
    const int rowB = p.WW * PB;
    const float wymax = static_cast<float>(p.WH - 2), wxmax = static_cast<float>(p.WW - 2);
    const int rowC = f.W * f.C;
    const float fdil = static_cast<float>(f.dilation);
    const int within = row_runs ? (px * f.G + gl) : gl;  // unit index inside its record run

    const int wslice = warp % p.tail_split;  // this warp's slice of a split tail tile
    for (int i = 0; i < ntiles; ++i) {
        int part;
        const unsigned t = item_tile(p, first + i * stride_t, &part);
        const bool my_slice = part < 0 || part == wslice;
        const int rb = i % nrec, wb = i & 1;
        bool ok = mbar_wait_bounded(&rec_full[rb], (i / nrec) & 1, kCopyWaitLimitNs);
        ok = ok && mbar_wait_bounded(&win_full[wb], (i >> 1) & 1, kCopyWaitLimitNs);
        if (!__all_sync(0xffffffffu, ok)) {
            if (lane == 0) atomicOr(&g_device_status, kStatusCopyTimeout);
            return;
        }
        const TileCoord c = tile_coord(p, t);
        if (has_unit && my_slice && py < c.nh && px < c.nw) {
            const unsigned char* win = winbuf + wb * p.win_bytes;
            const T* ximg = x + static_cast<size_t>(c.n) * f.H * rowC;
            const int ho = c.ho0 + py, wo = c.wo0 + px, g = c.gsub * p.GS + gl;

            // this unit's record in shared memory
            const int run = row_runs ? py : py * c.nw + px;
            int count;
            const unsigned long long ra = reinterpret_cast<unsigned long long>(run_src<T>(p, c, om, run, &count));
            const T* rec = reinterpret_cast<const T*>(recbuf + rb * p.rec_bytes + run * p.run_slot + (ra & 15)) +
                           within * R3;

            const unsigned char* ubase = win + gl * (Q * 16);
            float2 acc[Q][CH / 2];
#pragma unroll
            for (int j = 0; j < Q; ++j)
#pragma unroll
                for (int q = 0; q < CH / 2; ++q) acc[j][q] = make_float2(0.f, 0.f);

            const int by = ho * f.stride - f.pad;  // grid row of ky = 0 (image coordinates)
            const int bx = wo * f.stride - f.pad;
            const float fwy = static_cast<float>(by - c.wy0), fwx = static_cast<float>(bx - c.wx0);
            unsigned long long slow = 0ull;  // grid points left for the global-memory pass (K*K <= 64)
            const MaskNorm mn = VF ? mask_norm(rec + 2 * NP, NP, f.flags) : MaskNorm{0.f, 1.f, false};

#pragma unroll (KS > 0 ? KS * KS : 1)
            for (int k = 0; k < KK; ++k) {
                if (k == kcs) continue;
                const int jp = k - (k > kcs ? 1 : 0);  // point index in the record
                const int ky = k / K, kx = k - (k / K) * K;
                const float rx = ElemTraits<T>::to_float(rec[jp]);
                const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
                const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
                const float dy = __fmul_rn(f.offset_scale, ry);
                const float dx = __fmul_rn(f.offset_scale, rx);
                const float fy0 = floorf(dy), fx0 = floorf(dx);
                // window-relative top-left corner (exact: every term is a small integer)
                const float wyf = fy0 + (fwy + static_cast<float>(ky) * fdil);
                const float wxf = fx0 + (fwx + static_cast<float>(kx) * fdil);
                if (wyf >= 0.f && wyf <= wymax && wxf >= 0.f && wxf <= wxmax && fabsf(m) < INFINITY) {
                    // all four corners inside the window; outside-image corners read
                    // the window's zeros and the finite weight adds exactly 0
                    const float ly = dy - fy0, lx = dx - fx0;
                    const float a1 = m * ly, a0 = m - a1;          // m (1 - ly), m ly
                    const float w01 = a0 * lx, w00 = a0 - w01;    // a0 (1 - lx), a0 lx
                    const float w11 = a1 * lx, w10 = a1 - w11;
                    const int off = (static_cast<int>(wyf) * p.WW + static_cast<int>(wxf)) * PB;
                    const unsigned char* pb = ubase + off;
                    if constexpr (HW && std::is_same<T, __half>::value) {
                        const uint32_t wt = pack_half2(w00, w01), wbt = pack_half2(w10, w11);
#pragma unroll
                        for (int j = 0; j < Q; ++j) {
                            const unsigned char* pc = pb + (choff[j] << 4);
                            const uint4 v00 = *reinterpret_cast<const uint4*>(pc);
                            const uint4 v01 = *reinterpret_cast<const uint4*>(pc + PB);
                            const uint4 v10 = *reinterpret_cast<const uint4*>(pc + rowB);
                            const uint4 v11 = *reinterpret_cast<const uint4*>(pc + rowB + PB);
                            fma_chunk_h<false>(acc[j], wt, v00);
                            fma_chunk_h<true>(acc[j], wt, v01);
                            fma_chunk_h<false>(acc[j], wbt, v10);
                            fma_chunk_h<true>(acc[j], wbt, v11);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < Q; ++j) {
                            const unsigned char* pc = pb + (choff[j] << 4);
                            const uint4 v00 = *reinterpret_cast<const uint4*>(pc);
                            const uint4 v01 = *reinterpret_cast<const uint4*>(pc + PB);
                            const uint4 v10 = *reinterpret_cast<const uint4*>(pc + rowB);
                            const uint4 v11 = *reinterpret_cast<const uint4*>(pc + rowB + PB);
                            fma_chunk<T, HW>(acc[j], w00, v00);
                            fma_chunk<T, HW>(acc[j], w01, v01);
                            fma_chunk<T, HW>(acc[j], w10, v10);
                            fma_chunk<T, HW>(acc[j], w11, v11);
                        }
                    }
                } else {
                    slow |= 1ull << k;
                }
            }
            // the points outside the window: global gather with per-corner validity
            if constexpr (Q <= 2) {
                // two points per pass, so that their loads are in flight together
                while (slow) {
                    int kk[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        kk[h] = slow ? __ffsll(static_cast<long long>(slow)) - 1 : -1;
                        slow &= slow ? slow - 1ull : 0ull;
                    }
                    uint4 v[2][4][Q];
                    float w[2][4];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int k = kk[h] < 0 ? kk[0] : kk[h];
                        const int jp = k - (k > kcs ? 1 : 0);
                        const int ky = k / K, kx = k - (k / K) * K;
                        const float rx = ElemTraits<T>::to_float(rec[jp]);
                        const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
                        const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
                        Sample s = locate(by + ky * f.dilation, bx + kx * f.dilation, ry, rx, f.offset_scale, f.H, f.W);
                        if (kk[h] < 0) s.bits = 0u;
                        // the same weight arithmetic as the window path
                        const float a1 = m * s.ly, a0 = m - a1;
                        const float w01 = a0 * s.lx, w11 = a1 * s.lx;
                        w[h][0] = (s.bits & 1u) ? a0 - w01 : 0.f;
                        w[h][1] = (s.bits & 2u) ? w01 : 0.f;
                        w[h][2] = (s.bits & 4u) ? a1 - w11 : 0.f;
                        w[h][3] = (s.bits & 8u) ? w11 : 0.f;
                        const T* c00 = ximg + (s.y0 * f.W + s.x0) * f.C + g * f.Cg;
#pragma unroll
                        for (int cn = 0; cn < 4; ++cn) {
                            const bool in = (s.bits >> cn) & 1u;
                            const T* pcg = c00 + (cn >> 1) * rowC + (cn & 1) * f.C;
#pragma unroll
                            for (int j = 0; j < Q; ++j) {
                                uint32_t tt[4] = {0u, 0u, 0u, 0u};
                                if (in) load_vec<16>(pcg + choff[j] * CH, tt);
                                v[h][cn][j] = make_uint4(tt[0], tt[1], tt[2], tt[3]);
                            }
                        }
                    }
                    // corners outside the image (and a missing second point) carry
                    // weight 0 and x = 0, so they add exactly 0 whatever the mask holds
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int cn = 0; cn < 4; ++cn)
#pragma unroll
                            for (int j = 0; j < Q; ++j) fma_chunk<T, HW>(acc[j], w[h][cn], v[h][cn][j]);
                }
            } else {
                while (slow) {
                    const int k = __ffsll(static_cast<long long>(slow)) - 1;
                    slow &= slow - 1ull;
                    const int jp = k - (k > kcs ? 1 : 0);
                    const int ky = k / K, kx = k - (k / K) * K;
                    const float rx = ElemTraits<T>::to_float(rec[jp]);
                    const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
                    const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
                    const Sample s = locate(by + ky * f.dilation, bx + kx * f.dilation, ry, rx, f.offset_scale, f.H, f.W);
                    if (s.bits == 0u) continue;
                    // the same weight arithmetic as the window path
                    const float a1 = m * s.ly, a0 = m - a1;
                    const float w01 = a0 * s.lx, w11 = a1 * s.lx;
                    float w[4];
                    w[0] = (s.bits & 1u) ? a0 - w01 : 0.f;
                    w[1] = (s.bits & 2u) ? w01 : 0.f;
                    w[2] = (s.bits & 4u) ? a1 - w11 : 0.f;
                    w[3] = (s.bits & 8u) ? w11 : 0.f;
                    const T* c00 = ximg + (s.y0 * f.W + s.x0) * f.C + g * f.Cg;
#pragma unroll
                    for (int cn = 0; cn < 4; ++cn) {
                        if (!(s.bits & (1u << cn))) continue;
                        const T* pcg = c00 + (cn >> 1) * rowC + (cn & 1) * f.C;
#pragma unroll
                        for (int j = 0; j < Q; ++j) {
                            uint32_t tt[4];
                            load_vec<16>(pcg + choff[j] * CH, tt);
                            fma_chunk<T, HW>(acc[j], w[cn], make_uint4(tt[0], tt[1], tt[2], tt[3]));
                        }
                    }
                }
            }

            if (VF && (f.flags & kFlagCenterScale)) {
                // out = (1 - s) * aggregate + s * x at the centre grid position, read from the
                // window (which holds zeros outside the image)
                const float sg = center_gate<T>(f, (static_cast<size_t>((c.n * f.Hout + ho) * f.Wout + wo)) * f.G + g);
                const int cyw = by + (K / 2) * f.dilation - c.wy0, cxw = bx + (K / 2) * f.dilation - c.wx0;
                const unsigned char* pcx = ubase + (cyw * p.WW + cxw) * PB;
#pragma unroll
                for (int j = 0; j < Q; ++j) blend_chunk<T>(acc[j], sg, *reinterpret_cast<const uint4*>(pcx + (choff[j] << 4)));
            }
            T* o = out + (static_cast<size_t>((c.n * f.Hout + ho) * f.Wout + wo)) * f.C + g * f.Cg;
#pragma unroll
            for (int j = 0; j < Q; ++j) {
                const uint4 v = pack_chunk<T>(acc[j]);
                *reinterpret_cast<uint4*>(o + choff[j] * CH) = v;
            }
        }
        __syncwarp();
        if (lane == 0) {  // this warp is done with both buffers of tile i
            mbar_arrive(&rec_empty[rb]);
            mbar_arrive(&win_empty[wb]);
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
        fence_barrier_init();
        mbar_expect_tx(&bar, 16);
        mbar_arrive(&bar);
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(&g_device_status, kStatusSelftestTimeout);
    }
}

}  // namespace dcnv4
