// Ring-window kernel of the DCNv4 forward aggregation (sm_100a).
//
// The scattered 2x2 corner gathers are the whole cost of the op ("DCNv4：重塑视觉模型核心",
// bqwf.cn, section 2.2: memory access dominates). Served from L1 they return a
// couple of 32-byte sectors per clock; served from shared memory with a
// bank-aware layout they return a 128-byte wavefront per clock. So the kernel
// stages the input in shared memory and gathers from there.
//
// Work: a strip is one image, one band of TW output columns and one subset of
// GS channel groups. Strips are ordered (image, band, group subset) and their
// output rows one after the other ("strip-major"); every CTA (one per SM,
// persistent) takes one contiguous range of those rows, so CTAs differ by at
// most one output row of work. It walks its range in items of up to TH output
// rows.
//
// Shared memory holds a ring of NR input rows (window rows: TW output columns
// widened by the grid span and a halo of R pixels on each side, all GS*Cg
// channels of each pixel) plus one mirror row after them that repeats ring
// row 0, so a sample's lower corner row never needs a wrap test. Going down a
// strip, an item loads only the stride*rows its window gained; a new strip
// loads its whole window. Rows come by TMA tensor loads (cp.async.bulk.tensor,
// one input row each, no multicast; pixels outside the image arrive as zeros),
// the item's offset/mask records by bulk copies (one run per output row when
// the CTA owns every group, else one short run per pixel through 16-byte
// cp.async). A producer warp issues the copies as far ahead as the ring and
// the record buffers allow; consumer warps gather. Rows are reused while a
// strip continues, so every input row crosses L2 -> SM about
// WW / (TW * stride) times instead of once per overlapping tile.
//
// Thread <-> work: one thread per (pixel, group) unit of an item, covering all
// Cg channels of the unit as Q 16-byte chunks. Coordinates, corner indices and
// the four weights are computed once per (unit, point) and reused across the
// channels ("不只是卷积的平替", jsqmd.com, section 1: coefficient reuse and merged
// per-group channel work). A window pixel holds its GS*Cg channels
// contiguously (PB bytes); when PB is a multiple of 128 a chunk's bank quad
// does not depend on the pixel, and with each lane starting at a rotated chunk
// (rot) a quarter warp reads 8 distinct bank quads per LDS.128.
//
// Which samples are gathered from shared memory depends on the unit alone: a
// sample takes the window path when its 2x2 corners lie within R pixels of the
// unit's own K x K grid footprint (and its mask is finite); the others are
// gathered afterwards from global memory with per-corner validity. So the
// arithmetic of every output element, and its summation order, do not depend
// on how the rows are split among CTAs or items, nor on the batch size.
#pragma once

#include <cuda.h>

#include "dcnv4_async.cuh"
#include "dcnv4_kernels.cuh"

namespace dcnv4 {

struct RingParams {
    FwdParams f;
    int TH, TW;          // output rows per item (at most), output columns per band
    int GS, nsub;        // groups per strip, G / GS
    int R;               // halo (pixels) around a unit's grid footprint (unit windows)
    int img;             // 1: every window is its whole image plus a one-pixel border (image windows)
    int UH, UW;          // a unit's window: (K-1)*dilation + 2R + 1 rows and columns; image windows: H + 2, W + 2
    int WW;              // window columns: (TW-1)*stride + UW; image windows: W + 2
    int NR;              // ring rows (a mirror of ring row 0 follows them)
    int PB;              // bytes per window pixel: GS * Cg * sizeof(T)
    int rowB;            // ring row pitch: WW * PB rounded up to 128 bytes (TMA destinations stay aligned)
    int cblk;            // tensor-map channel blocks per group subset
    int bands;           // ceil(Wout / TW)
    int rows_total;      // N * bands * nsub * Hout: the strip-major rows shared out among CTAs
    int strip_cost;      // rows' worth of time a CTA spends entering a strip (its window load), >= 0
    int units;           // TH * TW * GS
    int run_slot;        // shared bytes per record run (an odd multiple of 16)
    int rec_bytes;       // one record buffer (multiple of 128)
    int ring_bytes;      // (NR + 1) * rowB rounded up to 128
    int nrec;            // record buffers = items in flight (2..4)
    unsigned long long om_lo, om_hi;  // byte range of the offset_mask tensor
    FastDiv div_tw_gs, div_gs, div_nsub, div_bands, div_hout;
    unsigned* status;    // device status word (bit kStatusCopyTimeout)
    int4* trace;         // tracing builds: per (unit, point) the corner, validity and path used
};

// ------------------------------------------------------------ chunk math ---

// Accumulates w * x over one 16-byte chunk (16/sizeof(T) channels) into acc
// (pairs of fp32 accumulators).
//  - HW (fp16 storage only): the weight is rounded once to fp16 and each
//    fp16 x fp16 product, exact in fp32, is added to the fp32 accumulator by
//    one mixed-precision FMA (fma.rn.f32.f16): no conversion of x.
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

// m times the four bilinear corner weights of a sample with fractional parts
// (ly, lx). For a finite m the window path's arithmetic: m ly, m (1 - ly) as
// m - m ly, and likewise along x, so that both paths give the same bits. For
// a non-finite m each corner's (m wy) wx, as in the plain definition: an
// infinite mask then gives +-Inf, or NaN where a weight is 0, per corner
// (m - m ly would be Inf - Inf = NaN for every corner).
__device__ __forceinline__ void corner_weights(float m, float ly, float lx, float& w00, float& w01, float& w10,
                                               float& w11) {
    if (fabsf(m) < INFINITY) {
        const float a1 = m * ly, a0 = m - a1;
        w01 = a0 * lx;
        w00 = a0 - w01;
        w11 = a1 * lx;
        w10 = a1 - w11;
    } else {
        const float b0 = m * (1.f - ly), b1 = m * ly;
        w00 = b0 * (1.f - lx);
        w01 = b0 * lx;
        w10 = b1 * (1.f - lx);
        w11 = b1 * lx;
    }
}

// 1.5 * 2^23 and its bit pattern: the floor of |d| < 2^22 by one directed add.
constexpr float kMagic = 12582912.0f;
constexpr unsigned kMagicBits = 0x4B400000u;

// 16-byte shared-memory load at a 32-bit shared-window address plus a
// compile-time byte offset. Ordered after the item's "full" wait by its data
// dependence: every address is computed from records read after that wait.
template <int OFF = 0>
__device__ __forceinline__ uint4 lds128(unsigned a) {
    uint4 v;
    asm("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4+%5];"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
        : "r"(a), "n"(OFF));
    return v;
}
__device__ __forceinline__ uint4 lds128r(unsigned a, unsigned off) { return lds128<0>(a + off); }

// Two fp32 weights to a pair of fp16 (round to nearest even), one instruction.
__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// acc += w * x over one fp16 chunk with mixed-precision FMAs; `w2` holds the
// fp16 weight in its low (HI == false) or high half.
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

// ------------------------------------------------------------ items ---

// One item of a CTA's row range, and where its window sits in the ring.
struct Item {
    int n, gsub, wo0, nw;   // image, group subset, first output column, columns
    int ho0, nh;            // first output row, rows
    int v, p0;              // window: first virtual ring row, its physical ring row
    int lv, lp, ln;         // rows to load: first virtual row, its physical row, count
};

// Walks a CTA's contiguous range of strip-major output rows. The producer and
// the consumers run identical cursors, so they agree on every item without
// communicating. Virtual ring rows count every row the CTA has loaded.
struct ItemCursor {
    int g, g1;               // next strip-major row, end of the range
    int strip, ho_end;       // last item's strip and the row after it (-1: none yet)
    int v, p0, nrows, adv;   // last item's window: virtual row, ring row, rows, advance to a continuation
};

// First strip-major row of the rows whose cost lies at or after `cost`, where
// the rows of strip s cost s (Hout + P) + P + (0 .. Hout - 1): every strip
// charges P rows' worth of time for entering it (its window load) before its
// rows. Monotonic, 0 at 0 and rows_total at the total cost.
__device__ __forceinline__ int row_at_cost(long long cost, int Hout, int P) {
    const long long per = static_cast<long long>(Hout) + P;
    const long long s = cost / per;
    const long long r = cost - s * per - P;
    return static_cast<int>(s * Hout + (r < 0 ? 0 : r));
}

// A CTA's contiguous range of strip-major rows: an equal share of the rows'
// total cost, so that a CTA whose range enters more strips gets fewer rows.
__device__ __forceinline__ ItemCursor item_cursor(const RingParams& p, int cta, int ncta) {
    ItemCursor c;
    const int Hout = p.f.Hout, P = p.strip_cost;
    const long long total = static_cast<long long>(p.rows_total / Hout) * (Hout + P);
    c.g = row_at_cost((total * cta) / ncta, Hout, P);
    c.g1 = row_at_cost((total * (cta + 1)) / ncta, Hout, P);
    c.strip = -1;
    c.ho_end = -1;
    c.v = 0;
    c.p0 = 0;
    c.nrows = 0;
    c.adv = 0;
    return c;
}

__device__ __forceinline__ bool next_item(const RingParams& p, ItemCursor& c, Item& it) {
    if (c.g >= c.g1) return false;
    const FwdParams& f = p.f;
    const int strip = static_cast<int>(fdiv(static_cast<unsigned>(c.g), p.div_hout));
    const int ho0 = c.g - strip * f.Hout;
    const int nh = min(p.TH, min(f.Hout - ho0, c.g1 - c.g));
    // an image window is the same for every item of its strip: loaded once, never advanced
    const int nrows = p.img ? p.UH : (nh - 1) * f.stride + p.UH;
    const bool cont = strip == c.strip && ho0 == c.ho_end;
    int v, p0;
    if (cont) {
        v = c.v + c.adv;
        p0 = c.p0 + c.adv;
    } else {
        v = c.v + c.nrows;
        p0 = c.p0 + c.nrows;
    }
    if (p0 >= p.NR) p0 -= p.NR;
    it.lv = cont ? c.v + c.nrows : v;
    int lp = cont ? c.p0 + c.nrows : p0;
    if (lp >= p.NR) lp -= p.NR;
    it.lp = lp;
    it.ln = v + nrows - it.lv;
    it.v = v;
    it.p0 = p0;
    it.ho0 = ho0;
    it.nh = nh;
    const unsigned s1 = fdiv(static_cast<unsigned>(strip), p.div_nsub);
    it.gsub = strip - static_cast<int>(s1) * p.nsub;
    const unsigned n = fdiv(s1, p.div_bands);
    const int band = static_cast<int>(s1 - n * p.bands);
    it.n = static_cast<int>(n);
    it.wo0 = band * p.TW;
    it.nw = min(p.TW, f.Wout - it.wo0);
    c.g += nh;
    c.strip = strip;
    c.ho_end = ho0 + nh;
    c.v = v;
    c.p0 = p0;
    c.nrows = nrows;
    c.adv = p.img ? 0 : nh * f.stride;
    return true;
}

// Address and element count of record run r of an item.
template <typename T>
__device__ __forceinline__ const unsigned char* run_src(const RingParams& p, const Item& it, const T* om, int r,
                                                        int* count) {
    const FwdParams& f = p.f;
    const bool row_runs = p.GS == f.G;
    const int py = row_runs ? r : r / it.nw;
    const int px = row_runs ? 0 : r - py * it.nw;
    const size_t first_unit = (static_cast<size_t>((it.n * f.Hout + it.ho0 + py) * f.Wout + it.wo0 + px)) * f.G +
                              static_cast<size_t>(it.gsub) * p.GS;
    *count = (row_runs ? it.nw * f.G : p.GS) * 3 * f.npts;
    return reinterpret_cast<const unsigned char*>(om + first_unit * 3 * f.npts);
}

// Arrivals the "full" barrier of an item waits for: the producer's lane 0, plus
// every producer lane's cp.async arrival when the records go per pixel.
__host__ __device__ __forceinline__ unsigned rec_full_arrivals(bool row_runs) { return row_runs ? 1u : 33u; }

// Producer warp: queues the copies of an item's offset/mask records into `buf`
// on `bar`. Runs are widened to 16-byte boundaries when that stays inside the
// offset_mask tensor (else the aligned middle is copied and the ragged ends by
// plain stores). An output row's records are one run and go by one bulk copy
// (cp.async.bulk). When the CTA owns only some of the groups the runs are per
// pixel and short; those go by 16-byte cp.async from all 32 lanes (a bulk copy
// costs the TMA unit tens of cycles each, too many for 100+ runs).
template <typename T>
__device__ __forceinline__ void issue_records(const RingParams& p, const T* om, const Item& it, unsigned char* buf,
                                              uint64_t* bar, int lane) {
    constexpr int E = sizeof(T);
    const bool row_runs = p.GS == p.f.G;
    const int nruns = row_runs ? it.nh : it.nh * it.nw;
    for (int r = lane; r < nruns; r += 32) {
        int count;
        const unsigned char* s = run_src<T>(p, it, om, r, &count);
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
}

// Producer warp: the window rows an item adds to the ring, one TMA row load
// each (spread over the lanes), plus the mirror row whenever ring row 0 is
// written.
__device__ __forceinline__ void issue_rows(const RingParams& p, const CUtensorMap* xmap, const Item& it,
                                           unsigned char* ring, uint64_t* bar, int lane) {
    const FwdParams& f = p.f;
    // image row and column of the window's first row and column
    const int img_top = p.img ? -1 : (it.ho0 + f.row0) * f.stride - f.pad - p.R;
    const int img_left = p.img ? -1 : it.wo0 * f.stride - f.pad - p.R;
    const int first = img_top + (it.lv - it.v);
    const unsigned box = static_cast<unsigned>(p.WW * p.PB);  // bytes of one row load
    for (int r = lane; r < it.ln; r += 32) {
        int phys = it.lp + r;
        if (phys >= p.NR) phys -= p.NR;
        const unsigned copies = phys == 0 ? 2u : 1u;
        mbar_expect_tx(bar, copies * box);
        tma_load_5d(ring + phys * p.rowB, xmap, 0, it.gsub * p.cblk, img_left, first + r, it.n, bar);
        if (phys == 0) tma_load_5d(ring + p.NR * p.rowB, xmap, 0, it.gsub * p.cblk, img_left, first + r, it.n, bar);
    }
}

// ------------------------------------------------------------ the kernel ---

// Warp roles: warps 0 .. nc-1 consume (gather), warp nc produces (issues the
// copies). Item i uses barrier/record slot i % nrec: its "full" barrier counts
// the producer's arrival(s) and the bytes of its rows and records; its "done"
// barrier one arrival per consumer warp. Before loading rows the producer
// waits until every item whose window still holds the ring rows they replace
// is done. No CTA-wide barrier is taken after the set-up. Every wait is
// bounded; a wait that gives up sets kStatusCopyTimeout in the status word and
// the warp leaves (the producer after letting its copies in flight land).
//
// VF: the variant flags of p.f may be set (softmax over the masks, centre
// point removed, centre feature scaling); false compiles them out.
// TRACE: also write, for every (unit, point), the top-left corner, the 4-bit
// validity and the path (0: shared-memory window, 1: global memory) that the
// gather used; compiled out of the forward's own builds.
// PBC: the window's pixel pitch as a compile-time constant (0: p.PB), so that
// the right-hand corners are immediate offsets of the left-hand ones.
// Registers: capped at 128 per thread with one or two 16-byte chunks per group
// (measured 1.5-2 % faster than 112 on the stage-1 fp16 and high-resolution
// bf16 workloads) and 112 otherwise (the 128 cap measured 1 % slower on
// stage-1 fp32); with at most 480 consumer threads per CTA each SM
// sub-partition (16 K registers) holds its 4 warps either way.
#ifndef DCNV4_RING_MAXREG
#define DCNV4_RING_MAXREG 112  // registers per thread with four or more chunks per group (build option)
#endif
#ifndef DCNV4_RING_MAXREG_NARROW
#define DCNV4_RING_MAXREG_NARROW 128  // registers per thread with one or two chunks per group
#endif
template <int Q>
constexpr int ring_maxreg() { return Q <= 2 ? DCNV4_RING_MAXREG_NARROW : DCNV4_RING_MAXREG; }

template <typename T, int Q, int KS, bool HW, int PBC, bool VF, bool TRACE>
__global__ void __maxnreg__(ring_maxreg<Q>())
fwd_ring_kernel(const __grid_constant__ CUtensorMap xmap, const T* __restrict__ x, const T* __restrict__ om,
                T* __restrict__ out, RingParams p) {
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[4], done[4];
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
    unsigned char* const ring = smem;                      // NR + 1 rows
    unsigned char* const recbuf = smem + p.ring_bytes;     // nrec record sets

    if (tid == 0) {
        for (int b = 0; b < 4; ++b) {
            mbar_init(&full[b], rec_full_arrivals(row_runs));
            mbar_init(&done[b], static_cast<unsigned>(nc));
        }
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&xmap)) : "memory");
    }
    __syncthreads();
    // Launched with programmatic stream serialisation, this grid may start while
    // the kernel before it on the stream is still running: wait for that grid to
    // complete (and its writes to be visible) before touching global memory,
    // then let the next launch on the stream start its own prologue as our SMs
    // free up. Without a programmatic dependency both return at once.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == nc) {
        // ---------------------------------------------------------------- producer
        ItemCursor cur = item_cursor(p, blockIdx.x, gridDim.x);
        // window start (virtual row) of the items in flight: vh0 is item d's, vh1 item d+1's, ...
        // (at most nrec <= 4 items are in flight; kept in registers, shifted as d advances)
        int vh0 = 0, vh1 = 0, vh2 = 0, vh3 = 0;
        int d = 0;  // items known to be done
        for (int i = 0;; ++i) {
            Item it;
            if (!next_item(p, cur, it)) break;
            // the rows below `need` (virtual) are overwritten; the record/barrier slot is item i - nrec's
            const int need = it.lv + it.ln - p.NR;
            bool ok = true;
            while (ok && d < i && (d <= i - nrec || vh0 < need)) {
                ok = mbar_wait_bounded(&done[d % nrec], (d / nrec) & 1, kCopyWaitLimitNs);
                ++d;
                vh0 = vh1; vh1 = vh2; vh2 = vh3;
            }
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) atomicOr(p.status, kStatusCopyTimeout);
                // let the copies already queued land before leaving
                for (int q = max(0, i - nrec); q < i; ++q)
                    mbar_wait_bounded(&full[q % nrec], (q / nrec) & 1, kCopyWaitLimitNs);
                return;
            }
            // item i is the (i - d)-th in flight
            const int slot = i - d;
            if (slot == 0) vh0 = it.v;
            else if (slot == 1) vh1 = it.v;
            else if (slot == 2) vh2 = it.v;
            else vh3 = it.v;
            fence_proxy_async();  // the consumers' reads of those buffers before the async writes
            issue_records<T>(p, om, it, recbuf + (i % nrec) * p.rec_bytes, &full[i % nrec], lane);
            issue_rows(p, &xmap, it, ring, &full[i % nrec], lane);
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[i % nrec]);
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    // this thread's unit (the same in every item) and its chunk rotation
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
        choff[j] = cc << 4;
    }
    const int rowB = p.rowB;
    const unsigned NR = static_cast<unsigned>(p.NR);
    // largest window row / column of a top-left corner
    const unsigned umy = static_cast<unsigned>(p.UH - 2), umx = static_cast<unsigned>(p.UW - 2);
    const bool img = p.img != 0;
    const int rowC = f.W * f.C;
    const int within = row_runs ? (px * f.G + gl) : gl;  // unit index inside its record run
    const unsigned char* const ubase = ring + gl * (Q * 16);
    const int cb = img ? 0 : px * f.stride;  // this unit's first window column
    // this lane's chunks of ring pixel (0, cb), in its rotated order (32-bit shared-window addresses)
    unsigned cbase_s[Q];
#pragma unroll
    for (int j = 0; j < Q; ++j) cbase_s[j] = smem_addr(ubase + choff[j] + cb * PB);
    const unsigned rowBu = static_cast<unsigned>(p.rowB), PBu = static_cast<unsigned>(PB);
    const unsigned ringB = NR * rowBu;  // bytes of the ring rows (the mirror row follows)

    ItemCursor cur = item_cursor(p, blockIdx.x, gridDim.x);
    for (int i = 0;; ++i) {
        Item it;
        if (!next_item(p, cur, it)) break;
        const int rb = i % nrec;
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&full[rb], (i / nrec) & 1, kCopyWaitLimitNs))) {
            if (lane == 0) atomicOr(p.status, kStatusCopyTimeout);
            return;
        }
        if (has_unit && py < it.nh && px < it.nw) {
            const int ho = it.ho0 + py, wo = it.wo0 + px, g = it.gsub * p.GS + gl;
            const T* ximg = x + static_cast<size_t>(it.n) * f.H * rowC;

            // this unit's record in shared memory (the run's copy starts at its address mod 16)
            const int run = row_runs ? py : py * it.nw + px;
            const unsigned first_unit = static_cast<unsigned>(
                ((it.n * f.Hout + ho) * f.Wout + it.wo0 + (row_runs ? 0 : px)) * f.G + it.gsub * p.GS);
            const unsigned shift = (static_cast<unsigned>(p.om_lo) + first_unit * static_cast<unsigned>(R3 * E)) & 15u;
            const T* rec = reinterpret_cast<const T*>(recbuf + rb * p.rec_bytes + run * p.run_slot + shift) +
                           within * R3;

            float2 acc[Q][CH / 2];
#pragma unroll
            for (int j = 0; j < Q; ++j)
#pragma unroll
                for (int q = 0; q < CH / 2; ++q) acc[j][q] = make_float2(0.f, 0.f);

            // ring row of this unit's window top, as a byte offset
            unsigned rb0 = static_cast<unsigned>(img ? it.p0 : it.p0 + py * f.stride);
            rb0 = min(rb0, rb0 - NR);
            const unsigned rowoff = rb0 * rowBu;
            const int by = (ho + f.row0) * f.stride - f.pad;  // grid row of ky = 0 (image coordinates)
            const int bx = wo * f.stride - f.pad;
            // window row / column of the grid point (0, 0): R in a unit window, which is
            // centred on the unit; in an image window (first row and column: image row and
            // column -1) the grid point's own image coordinates plus one
            const int cy = img ? by + 1 : p.R, cx = img ? bx + 1 : p.R;
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
                // floor without the conversion pipe: for |d| < 2^22, d + 1.5*2^23 rounded
                // toward -inf is exactly floor(d) + 1.5*2^23, a float whose bit pattern
                // minus kMagicBits is floor(d). Larger |d|, infinities and NaN give bit
                // patterns far outside the window's range below, so they take the global
                // pass (where floorf decides as everywhere else).
                const float ty = __fadd_rd(dy, kMagic), tx = __fadd_rd(dx, kMagic);
                // corner row / column inside the unit's window
                const unsigned uy = __float_as_uint(ty) + static_cast<unsigned>(ky * f.dilation + cy) - kMagicBits;
                const unsigned ux = __float_as_uint(tx) + static_cast<unsigned>(kx * f.dilation + cx) - kMagicBits;
                const bool inwin = uy <= umy && ux <= umx;
                if (inwin && fabsf(m) < INFINITY) {
                    // all four corners inside the window; outside-image corners read
                    // the window's zeros and the finite weight adds exactly 0
                    const float fy0 = ty - kMagic, fx0 = tx - kMagic;  // floor(dy), floor(dx), exact
                    const float ly = dy - fy0, lx = dx - fx0;
                    const float a1 = m * ly, a0 = m - a1;          // m ly, m (1 - ly)
                    const float w01 = a0 * lx, w00 = a0 - w01;    // a0 lx, a0 (1 - lx)
                    const float w11 = a1 * lx, w10 = a1 - w11;
                    // byte offset of the top-left corner in the ring (rows wrap once)
                    unsigned roff = rowoff + uy * rowBu;
                    roff = min(roff, roff - ringB);
                    const unsigned off = roff + ux * PBu;
                    if constexpr (TRACE) {
                        // the corner the ring address was formed from
                        const int y0 = by + ky * f.dilation + static_cast<int>(__float_as_uint(ty) - kMagicBits);
                        const int x0 = bx + kx * f.dilation + static_cast<int>(__float_as_uint(tx) - kMagicBits);
                        const bool vy0 = y0 >= 0 && y0 < f.H, vy1 = y0 + 1 >= 0 && y0 + 1 < f.H;
                        const bool vx0 = x0 >= 0 && x0 < f.W, vx1 = x0 + 1 >= 0 && x0 + 1 < f.W;
                        const int bits = (vy0 && vx0 ? 1 : 0) | (vy0 && vx1 ? 2 : 0) | (vy1 && vx0 ? 4 : 0) |
                                         (vy1 && vx1 ? 8 : 0);
                        const size_t ti = (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo) * f.G + g) * NP + jp;
                        p.trace[ti] = make_int4(bits ? y0 : INT_MIN, bits ? x0 : INT_MIN, bits, 0);
                    }
#pragma unroll
                    for (int j = 0; j < Q; ++j) {
                        const unsigned a = cbase_s[j] + off;
                        uint4 v00, v01, v10, v11;
                        if constexpr (PBC > 0) {
                            v00 = lds128<0>(a);
                            v01 = lds128<PBC>(a);
                            v10 = lds128r(a, rowBu);
                            v11 = lds128<PBC>(a + rowBu);
                        } else {
                            v00 = lds128<0>(a);
                            v01 = lds128r(a, PBu);
                            v10 = lds128r(a, rowBu);
                            v11 = lds128r(a, rowBu + PBu);
                        }
                        if constexpr (HW && std::is_same<T, __half>::value) {
                            const uint32_t wt = pack_half2(w00, w01), wbt = pack_half2(w10, w11);
                            fma_chunk_h<false>(acc[j], wt, v00);
                            fma_chunk_h<true>(acc[j], wt, v01);
                            fma_chunk_h<false>(acc[j], wbt, v10);
                            fma_chunk_h<true>(acc[j], wbt, v11);
                        } else {
                            fma_chunk<T, HW>(acc[j], w00, v00);
                            fma_chunk<T, HW>(acc[j], w01, v01);
                            fma_chunk<T, HW>(acc[j], w10, v10);
                            fma_chunk<T, HW>(acc[j], w11, v11);
                        }
                    }
                } else if (inwin || !img) {
                    slow |= 1ull << k;
                } else if constexpr (TRACE) {
                    // outside an image window: no corner lies inside the image, the
                    // sample adds nothing and is skipped
                    const size_t ti = (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo) * f.G + g) * NP + jp;
                    p.trace[ti] = make_int4(INT_MIN, INT_MIN, 0, 3);
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
                        if constexpr (TRACE) {
                            if (kk[h] >= 0) {
                                const size_t ti = (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo) * f.G + g) * NP + jp;
                                p.trace[ti] = make_int4(s.bits ? s.y0 : INT_MIN, s.bits ? s.x0 : INT_MIN,
                                                        static_cast<int>(s.bits), 1);
                            }
                        }
                        if (kk[h] < 0) s.bits = 0u;
                        // the same weight arithmetic as the window path
                        float v00, v01, v10, v11;
                        corner_weights(m, s.ly, s.lx, v00, v01, v10, v11);
                        w[h][0] = (s.bits & 1u) ? v00 : 0.f;
                        w[h][1] = (s.bits & 2u) ? v01 : 0.f;
                        w[h][2] = (s.bits & 4u) ? v10 : 0.f;
                        w[h][3] = (s.bits & 8u) ? v11 : 0.f;
                        const T* c00 = ximg + (s.y0 * f.W + s.x0) * f.C + g * f.Cg;
#pragma unroll
                        for (int cn = 0; cn < 4; ++cn) {
                            const bool in = (s.bits >> cn) & 1u;
                            const T* pcg = c00 + (cn >> 1) * rowC + (cn & 1) * f.C;
#pragma unroll
                            for (int j = 0; j < Q; ++j) {
                                uint32_t tt[4] = {0u, 0u, 0u, 0u};
                                if (in) load_vec<16>(reinterpret_cast<const unsigned char*>(pcg) + choff[j], tt);
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
                    if constexpr (TRACE) {
                        const size_t ti = (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo) * f.G + g) * NP + jp;
                        p.trace[ti] = make_int4(s.bits ? s.y0 : INT_MIN, s.bits ? s.x0 : INT_MIN,
                                                static_cast<int>(s.bits), 1);
                    }
                    if (s.bits == 0u) continue;
                    // the same weight arithmetic as the window path
                    float w[4];
                    corner_weights(m, s.ly, s.lx, w[0], w[1], w[2], w[3]);
                    const T* c00 = ximg + (s.y0 * f.W + s.x0) * f.C + g * f.Cg;
#pragma unroll
                    for (int cn = 0; cn < 4; ++cn) {
                        if (!(s.bits & (1u << cn))) continue;
                        const T* pcg = c00 + (cn >> 1) * rowC + (cn & 1) * f.C;
#pragma unroll
                        for (int j = 0; j < Q; ++j) {
                            uint32_t tt[4];
                            load_vec<16>(reinterpret_cast<const unsigned char*>(pcg) + choff[j], tt);
                            fma_chunk<T, HW>(acc[j], w[cn], make_uint4(tt[0], tt[1], tt[2], tt[3]));
                        }
                    }
                }
            }

            if (VF && (f.flags & kFlagCenterScale)) {
                // out = (1 - s) * aggregate + s * x at the centre grid position, read from the
                // window (which holds zeros outside the image)
                const float sg = center_gate<T>(f, (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo)) * f.G + g);
                // (an image window holds the centre only when the planner has checked so)
                const int cu = (K / 2) * f.dilation;
                unsigned t = rb0 + static_cast<unsigned>(cy + cu);
                t = min(t, t - NR);
                const unsigned char* pcx = ubase + static_cast<int>(t) * rowB + (cb + cx + cu) * PB;
#pragma unroll
                for (int j = 0; j < Q; ++j) blend_chunk<T>(acc[j], sg, *reinterpret_cast<const uint4*>(pcx + choff[j]));
            }
            T* o = out + (static_cast<size_t>((it.n * f.Hout + ho) * f.Wout + wo)) * f.C + g * f.Cg;
#pragma unroll
            for (int j = 0; j < Q; ++j) {
                const uint4 v = pack_chunk<T>(acc[j]);
                *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(o) + choff[j]) = v;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&done[rb]);  // this warp is done with item i's rows and records
    }
}

}  // namespace dcnv4
