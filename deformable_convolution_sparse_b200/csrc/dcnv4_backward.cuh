// sm_100a kernel of the DCNv4 backward: gradients of a loss with respect to
// the input x, the offsets and the masks, given the gradient of the output.
//
// The forward ("不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里",
// jsqmd.com, section 1) is out[c] = sum_k m_k * S_k[c] with S_k the zero-padded
// bilinear sample of x at grid point k moved by fl32(s * r). Its use for
// training (section 4 of the same page) needs, for dL/dout = go:
//   dL/dx at each in-bounds corner of each point  += m_k * W_corner * go[c]
//   dL/dm_k                                        = sum_c go[c] * S_k[c]
//   dL/dr (x part) = m_k * s * sum_c go[c] * dS_k[c]/dfx, likewise for y,
// with fx, fy the fractional parts of the sample position (S is linear in each
// of them inside a pixel cell; at an integer position the cell of floor(d) is
// used, as in the forward).
//
// Design (B200): like the forward, a gather that runs on the CUDA cores. A
// unit is one (pixel, group); `p.lanes` (a power of two <= 32) threads share
// it, each owning 4 of its channels per pass (one float4 of the gradient). Per point the four corner
// vectors are loaded once and give, per channel, the top and bottom row
// interpolants t and b: S = t + fy (b - t), dS/dfy = b - t and
// dS/dfx = (x01 - x00) + fy ((x11 - x10) - (x01 - x00)); the three channel
// sums are folded across the unit's lanes with xor shuffles. The x gradient is
// a scatter: each in-bounds corner gets m W go as fp32 vector reductions
// (`atomicAdd` on float4, resolved in L2), so its summation order, and only
// its, is not deterministic. These reductions bound the kernel: the requests
// they send from L1 to the L2 keep that path nearly saturated, so one warp
// instruction covers a unit's whole group slice of a corner (its lanes write
// adjacent float4s, which leave L1 as one request per 128-byte line).
// Accumulating a tile's contributions in shared memory first was tried and is
// several times slower: fp32 reductions into shared memory cost more than
// these L2 ones. The offset/mask gradient of the block's units is
// collected in shared memory and written out as one contiguous run.
#pragma once

#include "dcnv4_kernels.cuh"

namespace dcnv4 {

// locate() without the conversion pipe, for geometries whose grid positions
// and image sizes stay below 2^21 in magnitude (the caller checks; others call
// locate()). floor(d) of a scaled offset |d| < 2^22 is one directed add:
// d + 1.5*2^23 rounded toward -inf is exactly floor(d) + 1.5*2^23, whose bit
// pattern minus 0x4B400000 is floor(d). For larger offsets, infinities and NaN
// that difference (taken modulo 2^32) is at least 2^22 in magnitude, so every
// corner falls outside such an image, as in locate(). Inside, the corners,
// validity and fractional parts are locate()'s bit for bit.
__device__ __forceinline__ Sample locate_small(int p0y, int p0x, float ry, float rx, float scale, int H, int W) {
    constexpr float kMag = 12582912.0f;
    constexpr unsigned kMagBits = 0x4B400000u;
    Sample s;
    const float dy = __fmul_rn(scale, ry);
    const float dx = __fmul_rn(scale, rx);
    const float ty = __fadd_rd(dy, kMag), tx = __fadd_rd(dx, kMag);
    s.ly = dy - (ty - kMag);
    s.lx = dx - (tx - kMag);
    // y0 + 1 and x0 + 1 as unsigned: inside [0, H] x [0, W] iff some corner is in the image
    const unsigned uy = __float_as_uint(ty) - kMagBits + static_cast<unsigned>(p0y + 1);
    const unsigned ux = __float_as_uint(tx) - kMagBits + static_cast<unsigned>(p0x + 1);
    s.bits = 0u;
    s.y0 = 0;
    s.x0 = 0;
    if (uy <= static_cast<unsigned>(H) && ux <= static_cast<unsigned>(W)) {
        s.y0 = static_cast<int>(uy) - 1;
        s.x0 = static_cast<int>(ux) - 1;
        const bool vy0 = uy >= 1u, vy1 = uy + 1u <= static_cast<unsigned>(H);
        const bool vx0 = ux >= 1u, vx1 = ux + 1u <= static_cast<unsigned>(W);
        s.bits = (vy0 && vx0 ? 1u : 0u) | (vy0 && vx1 ? 2u : 0u) | (vy1 && vx0 ? 4u : 0u) | (vy1 && vx1 ? 8u : 0u);
    }
    return s;
}

// CPL channels of storage type T at p (8 or 16 bytes when CPL > 1) -> floats
template <typename T, int CPL>
__device__ __forceinline__ void load_channels(const T* p, float (&v)[CPL]) {
    if constexpr (CPL == 1) {
        v[0] = ElemTraits<T>::to_float(__ldg(p));
    } else if constexpr (CPL * sizeof(T) == 8) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(p));
        const float2 a = unpack2(w.x, static_cast<T*>(nullptr)), b = unpack2(w.y, static_cast<T*>(nullptr));
        v[0] = a.x;
        v[1] = a.y;
        v[2] = b.x;
        v[3] = b.y;
    } else {
        static_assert(CPL * sizeof(T) == 16, "vector chunks are 16 bytes");
        uint32_t w[4];
        load_vec<16>(p, w);
        if constexpr (sizeof(T) == 4) {
#pragma unroll
            for (int q = 0; q < 4; ++q) v[q] = __uint_as_float(w[q]);
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = unpack2(w[q], static_cast<T*>(nullptr));
                v[2 * q] = f.x;
                v[2 * q + 1] = f.y;
            }
        }
    }
}

// dst[0:CPL] += a * v[0:CPL] in fp32 global reductions (16-byte ones when CPL % 4 == 0)
template <int CPL>
__device__ __forceinline__ void scatter_add(float* dst, float a, const float (&v)[CPL]) {
    if constexpr (CPL % 4 == 0) {
#pragma unroll
        for (int q = 0; q < CPL; q += 4)
            atomicAdd(reinterpret_cast<float4*>(dst + q), make_float4(a * v[q], a * v[q + 1], a * v[q + 2], a * v[q + 3]));
    } else {
#pragma unroll
        for (int q = 0; q < CPL; ++q) atomicAdd(dst + q, a * v[q]);
    }
}

// grad_x must be zero on entry (the host clears it on the same stream);
// grad_om is overwritten. Shared memory: the block's records (T, staged at
// their 16-byte phase plus 16 bytes) followed, 16-byte aligned, by the block's
// fp32 gradient records.
//
// VF: the variant flags of p may be set (softmax over the masks, centre point
// removed, centre feature scaling); false compiles them out. With them, the
// aggregation part is the plain backward with masks m' (softmax-normalised or
// raw) and upstream (1 - s) dL/dout, s the centre gate; then the softmax's
// Jacobian maps dL/dm' to dL/dm, and centre scaling adds s dL/dout at the
// centre pixel of grad_x and writes dL/dz = s (1 - s) (sum_c g x_c -
// sum_j m'_j u_j), u_j = sum_c g S_j, to grad_z.
// LN: the lanes per unit as a compile-time constant when every lane owns
// exactly one chunk (p.chunks == p.lanes == LN; the fp32/fp16/bf16 16-channel
// groups: 4 lanes of 4 channels), 0 otherwise. With LN the lane's dL/dout
// chunk is loaded once per unit instead of once per point, and the chunk loop
// and the lane folds unroll.
template <typename T, int CPL, int KS, bool VF, int LN = 0>
__global__ void __launch_bounds__(256)
bwd_kernel(const T* __restrict__ x, const T* __restrict__ om, const T* __restrict__ go,
           float* __restrict__ grad_x, float* __restrict__ grad_om, float* __restrict__ grad_z, FwdParams p) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int K = KS > 0 ? KS : p.K;
    const int KK = K * K;
    const int NP = VF ? p.npts : KK;   // points per unit
    const int kcs = VF ? p.kc : KK;    // grid index left out (none: KK)
    const int R = 3 * NP;

    const int unit0 = blockIdx.x * p.units_per_block;
    const int nunits = min(p.units_per_block, p.units - unit0);
    const size_t rec_area = (static_cast<size_t>(p.units_per_block) * R * sizeof(T) + 16 + 15) & ~static_cast<size_t>(15);
    float* gbuf = reinterpret_cast<float*>(smem_raw + rec_area);
    const T* rec_base = stage_run<T>(om + static_cast<size_t>(unit0) * R, nunits * R, smem_raw);
    __syncthreads();

    const int lanes = LN > 0 ? LN : p.lanes;
    const int lu = threadIdx.x / lanes;
    const int part = threadIdx.x - lu * lanes;
    const bool active = lu < nunits;
    int n = 0, ho = 0, wo = 0, g = 0;
    if (active) unit_coords(unit0 + lu, p, n, ho, wo, g);
    const T* rec = rec_base + (active ? lu : 0) * R;

    const int rowC = p.W * p.C;
    const T* ximg = x + static_cast<size_t>(n) * p.H * rowC;
    float* gimg = grad_x + static_cast<size_t>(n) * p.H * rowC;
    const T* gop = go + (static_cast<size_t>((n * p.Hout + ho) * p.Wout + wo)) * p.C + g * p.Cg;
    const size_t unit = static_cast<size_t>(unit0 + (active ? lu : 0));
    const MaskNorm mn = VF ? mask_norm(rec + 2 * NP, NP, p.flags) : MaskNorm{0.f, 1.f, false};
    const bool cs = VF && (p.flags & kFlagCenterScale);
    const float sg = cs ? center_gate<T>(p, unit) : 0.f;   // centre gate s
    const float keep = 1.f - sg;                            // the aggregation's share of dL/dout
    float mu = 0.f;                                         // sum_j m'_j u_j (centre scaling)
    // locate_small() applies (LN builds): grid positions and image sizes below 2^21 in magnitude
    const bool small = LN > 0 &&
                       static_cast<long long>(p.Hout) * p.stride + p.pad + static_cast<long long>(p.K) * p.dilation +
                               p.H < (1LL << 21) &&
                       static_cast<long long>(p.Wout) * p.stride + p.pad + static_cast<long long>(p.K) * p.dilation +
                               p.W < (1LL << 21);
    float g1[CPL];                                          // LN: this lane's chunk of dL/dout
    if constexpr (LN > 0) {
        if (active) {
            load_channels<T, CPL>(gop + part * CPL, g1);
        } else {
#pragma unroll
            for (int q = 0; q < CPL; ++q) g1[q] = 0.f;
        }
    }

#pragma unroll (KS > 0 ? KS * KS : 1)
    for (int k = 0; k < KK; ++k) {
        if (k == kcs) continue;
        const int jp = k - (k > kcs ? 1 : 0);  // point index in the record
        const int ky = k / K, kx = k - (k / K) * K;
        const int p0y = ho * p.stride - p.pad + ky * p.dilation;
        const int p0x = wo * p.stride - p.pad + kx * p.dilation;
        const float rx = ElemTraits<T>::to_float(rec[jp]);
        const float ry = ElemTraits<T>::to_float(rec[NP + jp]);
        const float m = mask_value(ElemTraits<T>::to_float(rec[2 * NP + jp]), mn);
        Sample s = small ? locate_small(p0y, p0x, ry, rx, p.offset_scale, p.H, p.W)
                         : locate(p0y, p0x, ry, rx, p.offset_scale, p.H, p.W);
        if (!active) s.bits = 0u;

        float gm = 0.f, gfx = 0.f, gfy = 0.f;
        if (s.bits) {
            const float ly = s.ly, lx = s.lx;
            // mask times the corner weights, for the scatter into grad_x
            const float ms = VF ? m * keep : m;
            const float a1 = ms * ly, a0 = ms - a1;
            const float w01 = a0 * lx, w00 = a0 - w01, w11 = a1 * lx, w10 = a1 - w11;
            const float wc[4] = {w00, w01, w10, w11};
            // element offsets inside the image (LN builds: 32-bit, an image holds fewer
            // than 2^31 elements, checked on the host)
            using Off = typename std::conditional<(LN > 0), unsigned, size_t>::type;
            const Off c00 = static_cast<Off>(s.y0 * p.W + s.x0) * static_cast<Off>(p.C);
            const Off coff[4] = {c00, c00 + p.C, c00 + rowC, c00 + rowC + p.C};
            for (int ch = part; ch < (LN > 0 ? part + 1 : p.chunks); ch += lanes) {
                const int c0 = g * p.Cg + ch * CPL;
                float gv[CPL], xv[4][CPL];
                if constexpr (LN > 0) {
#pragma unroll
                    for (int q = 0; q < CPL; ++q) gv[q] = g1[q];
                } else {
                    load_channels<T, CPL>(gop + ch * CPL, gv);
                }
#pragma unroll
                for (int cn = 0; cn < 4; ++cn) {
                    if (s.bits & (1u << cn)) {
                        load_channels<T, CPL>(ximg + coff[cn] + c0, xv[cn]);
                    } else {
#pragma unroll
                        for (int q = 0; q < CPL; ++q) xv[cn][q] = 0.f;
                    }
                }
#pragma unroll
                for (int q = 0; q < CPL; ++q) {
                    const float d0 = xv[1][q] - xv[0][q];   // along x, top row
                    const float d1 = xv[3][q] - xv[2][q];   // along x, bottom row
                    const float t = fmaf(lx, d0, xv[0][q]);
                    const float b = fmaf(lx, d1, xv[2][q]);
                    const float dfy = b - t;
                    const float S = fmaf(ly, dfy, t);
                    const float dfx = fmaf(ly, d1 - d0, d0);
                    gm = fmaf(gv[q], S, gm);
                    gfy = fmaf(gv[q], dfy, gfy);
                    gfx = fmaf(gv[q], dfx, gfx);
                }
#pragma unroll
                for (int cn = 0; cn < 4; ++cn)
                    if (s.bits & (1u << cn)) scatter_add<CPL>(gimg + coff[cn] + c0, wc[cn], gv);
            }
        }
        // every lane of the warp reaches the folds (inactive lanes carry zeros)
        if constexpr (LN > 0) {
#pragma unroll
            for (int o = LN >> 1; o > 0; o >>= 1) {
                gm += __shfl_xor_sync(0xffffffffu, gm, o);
                gfx += __shfl_xor_sync(0xffffffffu, gfx, o);
                gfy += __shfl_xor_sync(0xffffffffu, gfy, o);
            }
        } else {
            for (int o = p.lanes >> 1; o > 0; o >>= 1) {
                gm += __shfl_xor_sync(0xffffffffu, gm, o);
                gfx += __shfl_xor_sync(0xffffffffu, gfx, o);
                gfy += __shfl_xor_sync(0xffffffffu, gfy, o);
            }
        }
        if (active && part == 0) {
            const float ms = (VF ? m * keep : m) * p.offset_scale;
            gbuf[lu * R + jp] = ms * gfx;
            gbuf[lu * R + NP + jp] = ms * gfy;
            gbuf[lu * R + 2 * NP + jp] = VF ? keep * gm : gm;   // dL/dm'
            if (VF) mu = fmaf(m, gm, mu);
        }
    }
    if constexpr (VF) {
        if (active && part == 0 && mn.on) {
            // softmax: dL/dm_j = m'_j (dL/dm'_j - sum_i m'_i dL/dm'_i)
            float* gmrow = gbuf + lu * R + 2 * NP;
            float dot = 0.f;
            for (int j = 0; j < NP; ++j) dot = fmaf(mask_value(ElemTraits<T>::to_float(rec[2 * NP + j]), mn), gmrow[j], dot);
            for (int j = 0; j < NP; ++j)
                gmrow[j] = mask_value(ElemTraits<T>::to_float(rec[2 * NP + j]), mn) * (gmrow[j] - dot);
        }
        if (cs) {
            // centre feature: grad_x[centre] += s g, and sum_c g x_c for the gate gradient
            const int cy = ho * p.stride - p.pad + (K / 2) * p.dilation;
            const int cx = wo * p.stride - p.pad + (K / 2) * p.dilation;
            const bool inside = active && cy >= 0 && cy < p.H && cx >= 0 && cx < p.W;
            float gxc = 0.f;
            if (inside) {
                const size_t cpix = static_cast<size_t>(cy * p.W + cx) * p.C;
                for (int ch = part; ch < p.chunks; ch += lanes) {
                    const int c0 = g * p.Cg + ch * CPL;
                    float gv[CPL], xv[CPL];
                    load_channels<T, CPL>(gop + ch * CPL, gv);
                    load_channels<T, CPL>(ximg + cpix + c0, xv);
#pragma unroll
                    for (int q = 0; q < CPL; ++q) gxc = fmaf(gv[q], xv[q], gxc);
                    scatter_add<CPL>(gimg + cpix + c0, sg, gv);
                }
            }
            for (int o = lanes >> 1; o > 0; o >>= 1) gxc += __shfl_xor_sync(0xffffffffu, gxc, o);
            if (active && part == 0) grad_z[unit] = sg * (1.f - sg) * (gxc - mu);
        }
    }
    __syncthreads();
    float* dst = grad_om + static_cast<size_t>(unit0) * R;
    for (int i = threadIdx.x; i < nunits * R; i += blockDim.x) dst[i] = gbuf[i];
}

}  // namespace dcnv4
