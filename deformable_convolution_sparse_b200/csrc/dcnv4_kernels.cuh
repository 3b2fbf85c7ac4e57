// sm_100a kernels of the DCNv4 forward spatial aggregation.
//
// Operation ("不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里", jsqmd.com,
// section 1, and its simplified forward listing): per output pixel and channel
// group, move each of the K*K regular grid points by its learned offset, sample
// the channels-last input bilinearly there (zero outside the image) and sum the
// samples weighted by the raw, un-normalised mask values.
//
// Design (B200): the op is a gather bounded by memory traffic, not a dense
// contraction, so it runs on the CUDA cores. One thread owns one (pixel, group)
// "unit" or a contiguous slice of its channels. The block's offset/mask records
// are one contiguous run of memory and are staged through shared memory with
// 16-byte loads. Corner indices, validity and the four bilinear weights (times
// the mask) are computed once per (unit, point) and reused across all the
// thread's channels (the "coefficient reuse" and "merged per-group channel
// work" of the pages, section 1). Channel slices are fetched with 128/256-bit
// read-only loads and accumulated in fp32 with packed f32x2 FMAs.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

namespace dcnv4 {

// Variant switches (the DCNV4_FLAG_* bits of the C ABI).
constexpr int kFlagSoftmax = 1;       // DCNv3: softmax over each unit's masks
constexpr int kFlagRemoveCenter = 2;  // K*K - 1 points: the centre grid point is left out
constexpr int kFlagCenterScale = 4;   // blend with the centre feature through a sigmoid gate

struct FwdParams {
    int N, H, W, C, G, K, KK, Cg;   // KK = K*K grid points
    int stride, pad, dilation;
    int Hout, Wout;     // output rows and columns of this launch (rows: of a band when row0 > 0)
    int row0;           // forward kernels: image row index of the launch's first output row, so that a
                        // launch can cover a band [row0, row0 + Hout) of each image's output rows (the
                        // offset_mask and out pointers then start at the band); 0 for whole images and
                        // for every other kernel
    int units;          // N * Hout * Wout * G
    int lanes;          // threads per unit
    int chunks;         // channel chunks per unit (a chunk is what one thread covers per pass)
    int units_per_block;
    float offset_scale;
    int npts;           // points per unit (record: 3 * npts elements): KK, or KK - 1 without the centre
    int kc;             // grid index left out (the centre), KK when none is
    int flags;          // kFlag* bits
    const void* center_logit;  // [N,Hout,Wout,G] gate logits (kFlagCenterScale), storage type of x
};

// ---------------------------------------------------------------- elements ---

template <typename T> struct ElemTraits;
template <> struct ElemTraits<float> {
    static __device__ __forceinline__ float to_float(float v) { return v; }
};
template <> struct ElemTraits<__half> {
    static __device__ __forceinline__ float to_float(__half v) { return __half2float(v); }
};
template <> struct ElemTraits<__nv_bfloat16> {
    static __device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }
};

// two storage elements packed in one 32-bit word -> two floats
__device__ __forceinline__ float2 unpack2(uint32_t w, __half*) {
    __half2 h = *reinterpret_cast<__half2*>(&w);
    return __half22float2(h);
}
__device__ __forceinline__ float2 unpack2(uint32_t w, __nv_bfloat16*) {
    // bf16 is the top half of an fp32 bit pattern
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __half*) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16*) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// a0 += w * x0; a1 += w * x1 as one packed fp32x2 FMA (two round-to-nearest FMAs)
__device__ __forceinline__ void fma2(float& a0, float& a1, float w, float x0, float x1) {
    asm("{\n\t.reg .b64 ra, rw, rx;\n\t"
        "mov.b64 ra, {%0, %1};\n\t"
        "mov.b64 rw, {%2, %2};\n\t"
        "mov.b64 rx, {%3, %4};\n\t"
        "fma.rn.f32x2 ra, rw, rx, ra;\n\t"
        "mov.b64 {%0, %1}, ra;\n\t}"
        : "+f"(a0), "+f"(a1)
        : "f"(w), "f"(x0), "f"(x1));
}

// ------------------------------------------------------------ vector memory ---

template <int VB> struct VecWords { static constexpr int n = VB / 4; };

template <int VB>
__device__ __forceinline__ void load_vec(const void* p, uint32_t (&w)[VB / 4]);

template <>
__device__ __forceinline__ void load_vec<16>(const void* p, uint32_t (&w)[4]) {
    asm("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
        : "l"(p));
}
template <>
__device__ __forceinline__ void load_vec<32>(const void* p, uint32_t (&w)[8]) {
    asm("ld.global.nc.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]),
          "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
        : "l"(p));
}

template <int VB>
__device__ __forceinline__ void store_vec(void* p, const uint32_t (&w)[VB / 4]);
template <>
__device__ __forceinline__ void store_vec<16>(void* p, const uint32_t (&w)[4]) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]) : "memory");
}
template <>
__device__ __forceinline__ void store_vec<32>(void* p, const uint32_t (&w)[8]) {
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                 :: "l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]),
                    "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]) : "memory");
}

// ------------------------------------------------------ record staging ---

// Copies `count` elements starting at `src` (any address aligned to sizeof(T))
// into shared memory. Element i lands at byte (src & 15) + i*sizeof(T) of
// `smem`, so that the aligned middle of the run moves with 16-byte loads and
// stores; the unaligned head and tail move element by element. Returns the
// shared-memory address of element 0. Every thread of the block must call it.
template <typename T>
__device__ __forceinline__ const T* stage_run(const T* __restrict__ src, int count, unsigned char* smem) {
    const uintptr_t a = reinterpret_cast<uintptr_t>(src);
    const int shift = static_cast<int>(a & 15);
    const int nbytes = count * static_cast<int>(sizeof(T));
    int head = (16 - shift) & 15;
    if (head > nbytes) head = nbytes;
    const int nvec = (nbytes - head) >> 4;
    const int tail0 = head + (nvec << 4);
    const unsigned char* s = reinterpret_cast<const unsigned char*>(src);
    unsigned char* d = smem + shift;
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(s + head) + i);
        *reinterpret_cast<uint4*>(d + head + (i << 4)) = v;
    }
    constexpr int E = sizeof(T);
    for (int i = threadIdx.x; i < head / E; i += blockDim.x)
        reinterpret_cast<T*>(d)[i] = src[i];
    for (int i = tail0 / E + threadIdx.x; i < count; i += blockDim.x)
        reinterpret_cast<T*>(d)[i] = src[i];
    return reinterpret_cast<const T*>(d);
}

// ------------------------------------------------------------ coordinates ---

// Integer and fractional parts of one sample, shared by every kernel so that
// the forward and the index dump agree bit for bit.
struct Sample {
    int y0, x0;     // top-left corner
    float ly, lx;   // fractional parts
    unsigned bits;  // corner validity: bit 2a+b for (y0+a, x0+b)
};

// dx, dy: raw stored offsets (already widened to fp32). The scaled offset is
// one round-to-nearest fp32 multiply; p0 + offset is never formed in floating
// point: floor(p0 + d) = p0 + floor(d) for integer p0.
__device__ __forceinline__ Sample locate(int p0y, int p0x, float ry, float rx, float scale, int H, int W) {
    Sample s;
    const float dy = __fmul_rn(scale, ry);
    const float dx = __fmul_rn(scale, rx);
    const float fy0 = floorf(dy), fx0 = floorf(dx);
    s.ly = dy - fy0;
    s.lx = dx - fx0;
    // some corner row is inside iff -1 <= p0y + floor(dy) <= H - 1; compared in
    // fp32 before any conversion (all bounds are exact: |p0| < 2^23), NaN fails
    const bool rows = (fy0 >= static_cast<float>(-1 - p0y)) && (fy0 <= static_cast<float>(H - 1 - p0y));
    const bool cols = (fx0 >= static_cast<float>(-1 - p0x)) && (fx0 <= static_cast<float>(W - 1 - p0x));
    s.bits = 0u;
    s.y0 = 0;
    s.x0 = 0;
    if (rows && cols) {
        s.y0 = p0y + static_cast<int>(fy0);
        s.x0 = p0x + static_cast<int>(fx0);
        const bool vy0 = s.y0 >= 0, vy1 = s.y0 + 1 <= H - 1;
        const bool vx0 = s.x0 >= 0, vx1 = s.x0 + 1 <= W - 1;
        s.bits = (vy0 && vx0 ? 1u : 0u) | (vy0 && vx1 ? 2u : 0u) |
                 (vy1 && vx0 ? 4u : 0u) | (vy1 && vx1 ? 8u : 0u);
    }
    return s;
}

// ------------------------------------------------------------ variants ---

// The masks a unit aggregates with: raw (DCNv4), or softmax-normalised over
// the unit's points (DCNv3, kFlagSoftmax): m'_j = exp(m_j - max) / sum.
struct MaskNorm {
    float mmax, inv;
    bool on;
};
template <typename T>
__device__ __forceinline__ MaskNorm mask_norm(const T* masks, int np, int flags) {
    MaskNorm r{0.f, 1.f, (flags & kFlagSoftmax) != 0};
    if (r.on) {
        float mx = -INFINITY;
        for (int j = 0; j < np; ++j) mx = fmaxf(mx, ElemTraits<T>::to_float(masks[j]));
        float sum = 0.f;
        for (int j = 0; j < np; ++j) sum += expf(ElemTraits<T>::to_float(masks[j]) - mx);
        r.mmax = mx;
        r.inv = 1.f / sum;
    }
    return r;
}
__device__ __forceinline__ float mask_value(float raw, const MaskNorm& n) {
    return n.on ? expf(raw - n.mmax) * n.inv : raw;
}

// Gate of the centre feature scaling: sigmoid of the unit's logit.
template <typename T>
__device__ __forceinline__ float center_gate(const FwdParams& p, size_t unit) {
    const float z = ElemTraits<T>::to_float(static_cast<const T*>(p.center_logit)[unit]);
    return 1.f / (1.f + expf(-z));
}

// Grid index of point j of a unit (the centre, when left out, is skipped).
__device__ __forceinline__ int grid_index(int j, int kc) { return j + (j >= kc ? 1 : 0); }

__device__ __forceinline__ void unit_coords(int unit, const FwdParams& p, int& n, int& ho, int& wo, int& g) {
    g = unit % p.G;
    int pix = unit / p.G;
    wo = pix % p.Wout;
    pix /= p.Wout;
    ho = pix % p.Hout;
    n = pix / p.Hout;
}

// ------------------------------------------------------ vector forward kernel ---

// One thread covers LB bytes (LB / VB vectors of VB bytes) of one unit's
// channels per pass; `p.lanes` threads share a unit and loop over
// `p.chunks` chunks. KS > 0 fixes K at compile time (0: runtime K). VF: the
// variant flags of p may be set (softmax over the masks, centre point
// removed, centre feature scaling); false compiles them out.
template <typename T, int VB, int LB, int KS, bool VF>
__global__ void __launch_bounds__(256)
fwd_vector_kernel(const T* __restrict__ x, const T* __restrict__ om, T* __restrict__ out, FwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    constexpr int E = sizeof(T);
    constexpr int NV = LB / VB;         // vectors per corner per thread
    constexpr int NW = LB / 4;          // 32-bit words per corner per thread
    constexpr int CPL = LB / E;         // channels per thread per pass
    const int K = KS > 0 ? KS : p.K;
    const int KK = K * K;
    const int NP = VF ? p.npts : KK;  // points per unit
    const int kcs = VF ? p.kc : KK;   // grid index left out (none: KK)
    const int R = 3 * NP;

    const int unit0 = blockIdx.x * p.units_per_block;
    const int nunits = min(p.units_per_block, p.units - unit0);
    const T* rec_base = stage_run<T>(om + static_cast<size_t>(unit0) * R, nunits * R, smem_raw);
    __syncthreads();

    const int lu = threadIdx.x / p.lanes;
    const int part = threadIdx.x - lu * p.lanes;
    if (lu >= nunits) return;
    const int unit = unit0 + lu;
    int n, ho, wo, g;
    unit_coords(unit, p, n, ho, wo, g);
    const T* rec = rec_base + lu * R;

    const int rowC = p.W * p.C;
    const T* ximg = x + static_cast<size_t>(n) * p.H * rowC;
    T* o = out + (static_cast<size_t>((n * p.Hout + ho) * p.Wout + wo)) * p.C + g * p.Cg;
    const MaskNorm mn = VF ? mask_norm(rec + 2 * NP, NP, p.flags) : MaskNorm{0.f, 1.f, false};

    for (int ch = part; ch < p.chunks; ch += p.lanes) {
        const int c0 = g * p.Cg + ch * CPL;   // first channel of this thread's slice
        float acc[CPL];
#pragma unroll
        for (int i = 0; i < CPL; ++i) acc[i] = 0.f;

#pragma unroll (KS > 0 ? KS * KS : 1)
        for (int k = 0; k < KK; ++k) {
            if (k == kcs) continue;
            const int jp = k - (k > kcs ? 1 : 0);  // point index in the record
            const int ky = k / K, kx = k - (k / K) * K;
            const int p0y = (ho + p.row0) * p.stride - p.pad + ky * p.dilation;
            const int p0x = wo * p.stride - p.pad + kx * p.dilation;
            const float rx = ElemTraits<T>::to_float(rec[jp]);
            const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
            const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
            const Sample s = locate(p0y, p0x, ry, rx, p.offset_scale, p.H, p.W);
            if (s.bits == 0u) continue;

            const float wy0 = 1.f - s.ly, wx0 = 1.f - s.lx;
            float w[4];
            w[0] = (s.bits & 1u) ? m * wy0 * wx0 : 0.f;
            w[1] = (s.bits & 2u) ? m * wy0 * s.lx : 0.f;
            w[2] = (s.bits & 4u) ? m * s.ly * wx0 : 0.f;
            w[3] = (s.bits & 8u) ? m * s.ly * s.lx : 0.f;

            const T* c00 = ximg + (s.y0 * p.W + s.x0) * p.C + c0;
            uint32_t v[4][NW];
#pragma unroll
            for (int cn = 0; cn < 4; ++cn) {
                const T* pc = c00 + ((cn >> 1) * rowC) + ((cn & 1) * p.C);
                if (s.bits & (1u << cn)) {
#pragma unroll
                    for (int j = 0; j < NV; ++j) {
                        uint32_t t[VB / 4];
                        load_vec<VB>(pc + j * (VB / E), t);
#pragma unroll
                        for (int q = 0; q < VB / 4; ++q) v[cn][j * (VB / 4) + q] = t[q];
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < NW; ++q) v[cn][q] = 0u;
                }
            }
#pragma unroll
            for (int cn = 0; cn < 4; ++cn) {
                if constexpr (E == 4) {
#pragma unroll
                    for (int q = 0; q < NW; q += 2)
                        fma2(acc[q], acc[q + 1], w[cn], __uint_as_float(v[cn][q]), __uint_as_float(v[cn][q + 1]));
                } else {
#pragma unroll
                    for (int q = 0; q < NW; ++q) {
                        const float2 f = unpack2(v[cn][q], static_cast<T*>(nullptr));
                        fma2(acc[2 * q], acc[2 * q + 1], w[cn], f.x, f.y);
                    }
                }
            }
        }

        if (VF && (p.flags & kFlagCenterScale)) {
            // out = (1 - s) * aggregate + s * x at the centre grid position (zero outside)
            const float sg = center_gate<T>(p, static_cast<size_t>(unit));
            const int cy = (ho + p.row0) * p.stride - p.pad + (K / 2) * p.dilation;
            const int cx = wo * p.stride - p.pad + (K / 2) * p.dilation;
            uint32_t cw[NW];
#pragma unroll
            for (int q = 0; q < NW; ++q) cw[q] = 0u;
            if (cy >= 0 && cy < p.H && cx >= 0 && cx < p.W) {
#pragma unroll
                for (int jv = 0; jv < NV; ++jv) {
                    uint32_t t[VB / 4];
                    load_vec<VB>(ximg + (cy * p.W + cx) * p.C + c0 + jv * (VB / E), t);
#pragma unroll
                    for (int q = 0; q < VB / 4; ++q) cw[jv * (VB / 4) + q] = t[q];
                }
            }
#pragma unroll
            for (int q = 0; q < NW; ++q) {
                if constexpr (E == 4) {
                    acc[q] = fmaf(sg, __uint_as_float(cw[q]), (1.f - sg) * acc[q]);
                } else {
                    const float2 f = unpack2(cw[q], static_cast<T*>(nullptr));
                    acc[2 * q] = fmaf(sg, f.x, (1.f - sg) * acc[2 * q]);
                    acc[2 * q + 1] = fmaf(sg, f.y, (1.f - sg) * acc[2 * q + 1]);
                }
            }
        }
        uint32_t ow[NW];
        if constexpr (E == 4) {
#pragma unroll
            for (int q = 0; q < NW; ++q) ow[q] = __float_as_uint(acc[q]);
        } else {
#pragma unroll
            for (int q = 0; q < NW; ++q) ow[q] = pack2(acc[2 * q], acc[2 * q + 1], static_cast<T*>(nullptr));
        }
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            uint32_t t[VB / 4];
#pragma unroll
            for (int q = 0; q < VB / 4; ++q) t[q] = ow[j * (VB / 4) + q];
            store_vec<VB>(o + ch * CPL + j * (VB / E), t);
        }
    }
}

// ------------------------------------------------------ scalar forward kernel ---

// Element-wise fallback for any channel count and alignment: one thread per
// (unit, channel) slot, looping over the unit's channels with stride p.lanes.
template <typename T, int KS, bool VF>
__global__ void __launch_bounds__(256)
fwd_scalar_kernel(const T* __restrict__ x, const T* __restrict__ om, T* __restrict__ out, FwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = KS > 0 ? KS : p.K;
    const int KK = K * K;
    const int NP = VF ? p.npts : KK;  // points per unit
    const int kcs = VF ? p.kc : KK;   // grid index left out (none: KK)
    const int R = 3 * NP;
    const int unit0 = blockIdx.x * p.units_per_block;
    const int nunits = min(p.units_per_block, p.units - unit0);
    const T* rec_base = stage_run<T>(om + static_cast<size_t>(unit0) * R, nunits * R, smem_raw);
    __syncthreads();

    const int lu = threadIdx.x / p.lanes;
    const int part = threadIdx.x - lu * p.lanes;
    if (lu >= nunits) return;
    const int unit = unit0 + lu;
    int n, ho, wo, g;
    unit_coords(unit, p, n, ho, wo, g);
    const T* rec = rec_base + lu * R;
    const int rowC = p.W * p.C;
    const T* ximg = x + static_cast<size_t>(n) * p.H * rowC;
    T* o = out + (static_cast<size_t>((n * p.Hout + ho) * p.Wout + wo)) * p.C + g * p.Cg;
    const MaskNorm mn = VF ? mask_norm(rec + 2 * NP, NP, p.flags) : MaskNorm{0.f, 1.f, false};

    for (int c = part; c < p.Cg; c += p.lanes) {
        float acc = 0.f;
        for (int k = 0; k < KK; ++k) {
            if (k == kcs) continue;
            const int jp = k - (k > kcs ? 1 : 0);  // point index in the record
            const int ky = k / K, kx = k - (k / K) * K;
            const int p0y = (ho + p.row0) * p.stride - p.pad + ky * p.dilation;
            const int p0x = wo * p.stride - p.pad + kx * p.dilation;
            const float rx = ElemTraits<T>::to_float(rec[jp]);
            const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
            const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
            const Sample s = locate(p0y, p0x, ry, rx, p.offset_scale, p.H, p.W);
            if (s.bits == 0u) continue;
            const float wy0 = 1.f - s.ly, wx0 = 1.f - s.lx;
            const T* c00 = ximg + (s.y0 * p.W + s.x0) * p.C + g * p.Cg + c;
            if (s.bits & 1u) acc = fmaf(m * wy0 * wx0, ElemTraits<T>::to_float(c00[0]), acc);
            if (s.bits & 2u) acc = fmaf(m * wy0 * s.lx, ElemTraits<T>::to_float(c00[p.C]), acc);
            if (s.bits & 4u) acc = fmaf(m * s.ly * wx0, ElemTraits<T>::to_float(c00[rowC]), acc);
            if (s.bits & 8u) acc = fmaf(m * s.ly * s.lx, ElemTraits<T>::to_float(c00[rowC + p.C]), acc);
        }
        if (VF && (p.flags & kFlagCenterScale)) {
            const float sg = center_gate<T>(p, static_cast<size_t>(unit));
            const int cy = (ho + p.row0) * p.stride - p.pad + (K / 2) * p.dilation;
            const int cx = wo * p.stride - p.pad + (K / 2) * p.dilation;
            const float xc = (cy >= 0 && cy < p.H && cx >= 0 && cx < p.W)
                                 ? ElemTraits<T>::to_float(ximg[(cy * p.W + cx) * p.C + g * p.Cg + c]) : 0.f;
            acc = fmaf(sg, xc, (1.f - sg) * acc);
        }
        if constexpr (sizeof(T) == 4) o[c] = acc;
        else if constexpr (std::is_same<T, __half>::value) o[c] = __float2half_rn(acc);
        else o[c] = __float2bfloat16_rn(acc);
    }
}

// ------------------------------------------------------ sampling-index kernel ---

// One thread per sampling point: writes (y0, x0) and the validity bits, using
// the same `locate` as the forward kernels.
template <typename T>
__global__ void __launch_bounds__(256)
sampling_index_kernel(const T* __restrict__ om, int32_t* __restrict__ corner, uint8_t* __restrict__ valid,
                      FwdParams p) {
    const int KK = p.KK;
    const long long total = static_cast<long long>(p.units) * KK;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int unit = static_cast<int>(i / KK);
        const int k = static_cast<int>(i - static_cast<long long>(unit) * KK);
        int n, ho, wo, g;
        unit_coords(unit, p, n, ho, wo, g);
        const T* rec = om + static_cast<size_t>(unit) * 3 * KK;
        const int ky = k / p.K, kx = k - (k / p.K) * p.K;
        const int p0y = (ho + p.row0) * p.stride - p.pad + ky * p.dilation;
        const int p0x = wo * p.stride - p.pad + kx * p.dilation;
        const Sample s = locate(p0y, p0x, ElemTraits<T>::to_float(rec[KK + k]), ElemTraits<T>::to_float(rec[k]),
                                p.offset_scale, p.H, p.W);
        valid[i] = static_cast<uint8_t>(s.bits);
        corner[2 * i] = s.bits ? s.y0 : INT32_MIN;
        corner[2 * i + 1] = s.bits ? s.x0 : INT32_MIN;
    }
}

// Trace of the global-gather kernel's sampling (a shape the ring kernel does not
// take): per sampling point (y0, x0, validity bits, path 2), computed by the
// same `locate` that kernel uses.
template <typename T>
__global__ void __launch_bounds__(256)
trace_index_kernel(const T* __restrict__ om, int4* __restrict__ trace, FwdParams p) {
    const int KK = p.KK;
    const long long total = static_cast<long long>(p.units) * KK;
    for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int unit = static_cast<int>(i / KK);
        const int k = static_cast<int>(i - static_cast<long long>(unit) * KK);
        int n, ho, wo, g;
        unit_coords(unit, p, n, ho, wo, g);
        const T* rec = om + static_cast<size_t>(unit) * 3 * KK;
        const int ky = k / p.K, kx = k - (k / p.K) * p.K;
        const Sample s = locate((ho + p.row0) * p.stride - p.pad + ky * p.dilation,
                                wo * p.stride - p.pad + kx * p.dilation, ElemTraits<T>::to_float(rec[KK + k]),
                                ElemTraits<T>::to_float(rec[k]), p.offset_scale, p.H, p.W);
        trace[i] = make_int4(s.bits ? s.y0 : INT32_MIN, s.bits ? s.x0 : INT32_MIN, static_cast<int>(s.bits), 2);
    }
}

}  // namespace dcnv4
