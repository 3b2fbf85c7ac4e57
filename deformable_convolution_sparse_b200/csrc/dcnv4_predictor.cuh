// sm_100a kernel of the DCNv4 offset/mask predictor's last step: the 1x1
// projection of the block's parameter network as a tensor-core GEMM whose
// epilogue writes the packed offset_mask records.
//
// "不只是卷积的平替：我把DCNv4塞进Stable Diffusion的U-Net里" (jsqmd.com), section 2:
// the block predicts its parameters with a depthwise 3x3 convolution followed
// by a 1x1 convolution to 3*groups*9 channels, the first 2*groups*9 being the
// offsets and the rest the masks (section 1's listing reshapes them as
// (N, G, 2, K*K, ...) and (N, G, K*K, ...)); it merges the two into one
// sub-network to cut memory traffic. Here the 1x1 convolution on channels-last
// activations y [M pixels, C] with weights W [NO = 3*G*P, C] is
//   params[m, o] = bias[o] + sum_c W[o, c] y[m, c]
// and the epilogue scatters params[m, :] into the record layout the
// aggregation reads: record[m, g, :] = [P x-offsets | P y-offsets | P masks].
//
// Design (B200, tcgen05): persistent CTAs, one per SM, each owning tiles of 128
// pixels. Warp 0 (one lane) issues TMA loads: W once (all C/64 k-blocks, rows
// padded to the MMA's N with the TMA's zero fill), then the 128 x C activation
// tile of every owned tile into a ring of `stages` buffers, 128-byte swizzled.
// Warp 1 (one lane) issues tcgen05.mma (M = 128, N = NP = NO rounded up to 16,
// K = 16 per instruction, fp32 accumulators in tensor memory, two accumulator
// buffers) and commits each tile to mbarriers that free its activation stage
// and hand its accumulator to the epilogue. The epilogue warps (EPW / 4 per
// 32-lane quarter of tensor memory, interleaved 16-column chunks) read their rows with tcgen05.ld
// (up to four loads in flight per wait), add the bias, round to the
// storage type, place every channel at its record slot in a shared-memory
// staging tile, and one thread writes the tile -- 128 consecutive records,
// one contiguous run of global memory -- with a bulk copy. Every wait is
// bounded; a wait that gives up sets the device status word and the CTA winds
// down (tensor memory is always released).
//
// Shapes: fp16 or bf16, C a multiple of 64 (one 128-byte swizzle atom per
// k-block), NO <= 256. Anything else takes the plain CUDA-core kernel below.
#pragma once

#include <cuda.h>

#include "dcnv4_async.cuh"
#include "dcnv4_kernels.cuh"

namespace dcnv4 {

struct PredParams {
    int M;          // pixels
    int C;          // input channels (multiple of 64 on the tensor-core path)
    int G, P;       // groups, points per group
    int NO;         // output channels 3*G*P
    int NP;         // NO rounded up to a multiple of 16 (the MMA's N)
    int tiles;      // ceil(M / 128)
    int kblocks;    // C / 64
    int stages;     // activation ring depth
    unsigned tmem_cols;  // tensor-memory columns allocated (power of two >= 2*NP)
    int a_fmt;      // 0: fp16, 1: bf16 (instruction-descriptor format code)
    int out_bufs;   // output staging buffers (2, or 1 when two do not fit)
    int w_in_staging;  // raw W fits the (still idle) output staging area: the activation loads start at once
    unsigned smem_b, smem_a, smem_o, smem_meta;  // byte offsets of the shared-memory regions
    unsigned* status;  // device status word (bit kStatusCopyTimeout)
};

// slot of projection channel o in its record: offsets (g, comp, j) -> g*3P + comp*P + j,
// masks (g, j) -> g*3P + 2P + j
__host__ __device__ __forceinline__ int pred_dest(int o, int G, int P) {
    if (o < 2 * G * P) return (o / (2 * P)) * 3 * P + o % (2 * P);
    const int q = o - 2 * G * P;
    return (q / P) * 3 * P + 2 * P + q % P;
}

// ---------------------------------------------------------------- tcgen05 ---

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_addr(bar))
        : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored in 128-byte
// swizzled atoms of 8 rows x 128 bytes (the TMA's SWIZZLE_128B layout):
// start address >> 4, leading offset 1 (unused for this layout), stride 1024
// bytes between 8-row atoms, descriptor version 1, layout code 2 (128-byte
// swizzle).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(unsigned saddr) {
    uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation, both operands
// K-major, M = 128, N = n.
__device__ __forceinline__ uint32_t mma_idesc(int fmt, int n) {
    return (1u << 4) | (static_cast<uint32_t>(fmt) << 7) | (static_cast<uint32_t>(fmt) << 10) |
           (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    const uint32_t z = 0u;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(z), "r"(z), "r"(z), "r"(z)
        : "memory");
}
// arrive on `bar` once every tcgen05.mma this thread issued so far has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's tensor-memory lane; the values
// are valid only after tmem_wait_ld()
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, float (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
          "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// named barrier over `count` threads that also returns the AND of every thread's `pred`
__device__ __forceinline__ bool named_bar_and(int id, int count, bool pred) {
    unsigned r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(count)
        : "memory");
    return r != 0;
}

template <typename T>
__device__ __forceinline__ T from_float(float v) {
    if constexpr (std::is_same<T, __half>::value) return __float2half_rn(v);
    else return __float2bfloat16_rn(v);
}

// 64 + 32 * EPW threads: warp 0 loads, warp 1 issues the MMAs, EPW epilogue
// warps (a multiple of 4: EPW / 4 per 32-lane quarter of tensor memory).
template <typename T, int EPW>
__global__ void __launch_bounds__(64 + 32 * EPW, 1)
predictor_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                    const float* __restrict__ bias, T* __restrict__ rec, PredParams p) {
    extern __shared__ unsigned char pred_smem_raw[];
    // 1024-byte alignment for the swizzled operand tiles
    unsigned char* sm = pred_smem_raw + ((1024u - (smem_addr(pred_smem_raw) & 1023u)) & 1023u);
    unsigned char* bsm = sm + p.smem_b;
    unsigned char* asm_ = sm + p.smem_a;
    T* osm = reinterpret_cast<T*>(sm + p.smem_o);
    int* src = reinterpret_cast<int*>(sm + p.smem_meta);      // projection channel of each record slot
    float* bias_s = reinterpret_cast<float*>(src + p.NO);     // bias in record order
    uint64_t* bars = reinterpret_cast<uint64_t*>(
        (reinterpret_cast<uintptr_t>(bias_s + p.NO) + 7) & ~static_cast<uintptr_t>(7));
    uint64_t* a_full = bars;
    uint64_t* a_empty = bars + p.stages;
    uint64_t* b_full = bars + 2 * p.stages;
    uint64_t* acc_full = b_full + 1;
    uint64_t* acc_empty = acc_full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    constexpr int E = sizeof(T);
    const unsigned a_stage_bytes = static_cast<unsigned>(p.kblocks) * 128u * 128u;
    const unsigned b_kblock_bytes = static_cast<unsigned>(p.NP) * 128u;
    const int ntiles = p.tiles > static_cast<int>(blockIdx.x)
                           ? (p.tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                                 static_cast<int>(gridDim.x)
                           : 0;

    if (tid == 0) {
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&a_full[s], 1);
            mbar_init(&a_empty[s], 1);
        }
        mbar_init(b_full, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 32 * EPW);
        }
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&amap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&bmap)) : "memory");
    }
    if (warp == 0) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(tmem_slot)),
                     "r"(p.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Launched with programmatic stream serialisation: wait for the previous
    // kernel on the stream (complete, its writes visible) before the first
    // global access, then let the next launch start its set-up as SMs free up.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int o = tid; o < p.NO; o += blockDim.x) {
        const int d = pred_dest(o, p.G, p.P);
        src[d] = o;
        bias_s[d] = bias ? bias[o] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // W, once per CTA: TMA into an idle area (the output staging tiles when it
    // fits there, else the activation ring), then its rows copied into record
    // order in bsm, so that accumulator column d is record slot d. Rows past NO
    // are the TMA's zero fill. A 16-byte chunk j of row r sits at chunk
    // j ^ (r mod 8) of the row (128-byte swizzle, 1024-byte atoms). Each "full"
    // barrier completes on one arrival plus the bytes of its loads. With W in
    // the staging area the first activation tiles are requested at once too.
    unsigned char* wraw = p.w_in_staging ? reinterpret_cast<unsigned char*>(osm) : asm_;
    const int preissued = (p.w_in_staging && ntiles > 0) ? min(p.stages, ntiles) : 0;
    if (tid == 0 && ntiles > 0) {
        mbar_expect_tx(b_full, static_cast<unsigned>(p.kblocks) * b_kblock_bytes);
        for (int kb = 0; kb < p.kblocks; ++kb) tma_load_2d(wraw + kb * b_kblock_bytes, &bmap, kb * 64, 0, b_full);
        mbar_arrive(b_full);
        for (int it = 0; it < preissued; ++it) {
            const int tile = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
            mbar_expect_tx(&a_full[it], a_stage_bytes);
            for (int kb = 0; kb < p.kblocks; ++kb)
                tma_load_2d(asm_ + it * a_stage_bytes + kb * 16384u, &amap, kb * 64, tile * 128, &a_full[it]);
            mbar_arrive(&a_full[it]);
        }
    }
    const bool b_ok = __syncthreads_and(ntiles == 0 || mbar_wait_bounded(b_full, 0u, kCopyWaitLimitNs)) != 0;
    if (b_ok && ntiles > 0) {
        const int items = p.kblocks * p.NP * 8;
        for (int i = tid; i < items; i += blockDim.x) {
            const int kb = i / (p.NP * 8), r = (i >> 3) % p.NP, j = i & 7;
            const int o = r < p.NO ? src[r] : r;
            const unsigned char* from = wraw + kb * b_kblock_bytes + (o >> 3) * 1024 + (o & 7) * 128 + ((j ^ (o & 7)) << 4);
            unsigned char* to = bsm + kb * b_kblock_bytes + (r >> 3) * 1024 + (r & 7) * 128 + ((j ^ (r & 7)) << 4);
            *reinterpret_cast<uint4*>(to) = *reinterpret_cast<const uint4*>(from);
        }
        fence_proxy_async();  // the generic writes of W, before the tensor cores read them
    }
    __syncthreads();
    if (!b_ok && tid == 0) atomicOr(p.status, kStatusCopyTimeout);

    if (!b_ok) {
        // nothing was started: straight to the release of tensor memory
    } else if (warp == 0) {
        if (lane == 0 && ntiles > 0) {
            // -------------------------------------------------------- loads
            for (int it = preissued; it < ntiles; ++it) {
                const int s = it % p.stages;
                if (it >= p.stages &&
                    !mbar_wait_bounded(&a_empty[s], static_cast<unsigned>((it / p.stages) - 1) & 1u, kCopyWaitLimitNs)) {
                    atomicOr(p.status, kStatusCopyTimeout);
                    break;
                }
                const int tile = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
                mbar_expect_tx(&a_full[s], a_stage_bytes);
                for (int kb = 0; kb < p.kblocks; ++kb)
                    tma_load_2d(asm_ + s * a_stage_bytes + kb * 16384u, &amap, kb * 64, tile * 128, &a_full[s]);
                mbar_arrive(&a_full[s]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && ntiles > 0) {
            // -------------------------------------------------------- MMAs
            const uint32_t idesc = mma_idesc(p.a_fmt, p.NP);
            bool ok = true;
            for (int it = 0; ok && it < ntiles; ++it) {
                const int s = it % p.stages, b = it & 1;
                if (it >= 2) ok = mbar_wait_bounded(&acc_empty[b], static_cast<unsigned>((it >> 1) - 1) & 1u,
                                                    kCopyWaitLimitNs);
                ok = ok && mbar_wait_bounded(&a_full[s], static_cast<unsigned>(it / p.stages) & 1u, kCopyWaitLimitNs);
                if (!ok) break;
                tc_fence_after();
                const uint32_t d = tmem_base + static_cast<uint32_t>(b * p.NP);
                const unsigned abase = smem_addr(asm_ + s * a_stage_bytes), bbase = smem_addr(bsm);
                for (int kb = 0; kb < p.kblocks; ++kb)
#pragma unroll
                    for (int k16 = 0; k16 < 4; ++k16) {
                        const uint64_t ad = sw128_kmajor_desc(abase + kb * 16384u + k16 * 32u);
                        const uint64_t bd = sw128_kmajor_desc(bbase + kb * b_kblock_bytes + k16 * 32u);
                        umma_f16(d, ad, bd, idesc, (kb | k16) != 0 ? 1u : 0u);
                    }
                umma_commit(&a_empty[s]);
                umma_commit(&acc_full[b]);
            }
            if (!ok) atomicOr(p.status, kStatusCopyTimeout);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        constexpr int NE = 32 * EPW;              // epilogue threads
        constexpr int EPQ = EPW / 4;              // epilogue warps per quarter
        const int et = tid - 64;                  // 0 .. NE-1
        const int quarter = warp & 3;             // tensor-memory lanes 32*quarter .. +31
        const int part = (warp - 2) >> 2;         // which 16-column chunks: part, part + EPQ, ...
        const int row = quarter * 32 + lane;      // row of the tile (pixel)
        const int nch = p.NP / 16;
        const size_t rec_tile = static_cast<size_t>(128) * p.NO;  // elements per full tile
        for (int it = 0; it < ntiles; ++it) {
            const int b = it & 1, ob_i = p.out_bufs == 2 ? b : 0;
            const int tile = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
            T* ob = osm + ob_i * rec_tile;
            // the bulk store that last read this staging buffer is done
            if (et == 0) {
                if (p.out_bufs == 2) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                else asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
            const bool ok = mbar_wait_bounded(&acc_full[b], static_cast<unsigned>(it >> 1) & 1u, kCopyWaitLimitNs);
            // one decision for all epilogue threads, so that they leave together
            if (!named_bar_and(1, NE, ok)) {
                if (et == 0) atomicOr(p.status, kStatusCopyTimeout);
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(b * p.NP);
            T* orow = ob + static_cast<size_t>(row) * p.NO;
            // up to four 16-column loads in flight before one wait
            for (int c = part; c < nch; c += 4 * EPQ) {
                float v[4][16];
                int n = 0;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int cc = c + EPQ * q;
                    if (cc < nch) {
                        tmem_ld16_nowait(taddr + static_cast<uint32_t>(cc * 16), v[q]);
                        n = q + 1;
                    }
                }
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (q >= n) break;
                    const int c0 = (c + EPQ * q) * 16;  // columns are record slots
                    if (p.NO % 2 == 0) {
                        // pairs of slots as one 32-bit store (row * NO and c0 are even)
#pragma unroll
                        for (int jj = 0; jj < 16; jj += 2) {
                            const int d = c0 + jj;
                            if (d < p.NO)
                                *reinterpret_cast<uint32_t*>(orow + d) =
                                    pack2(v[q][jj] + bias_s[d], v[q][jj + 1] + bias_s[d + 1], static_cast<T*>(nullptr));
                        }
                    } else {
#pragma unroll
                        for (int jj = 0; jj < 16; ++jj) {
                            const int d = c0 + jj;
                            if (d < p.NO) orow[d] = from_float<T>(v[q][jj] + bias_s[d]);
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[b]);
            fence_proxy_async();  // the staging writes, before the bulk copy reads them
            named_bar_sync(1, NE);
            const int rows = min(128, p.M - tile * 128);
            T* gdst = rec + static_cast<size_t>(tile) * rec_tile;
            if (rows == 128) {
                if (et == 0) {
                    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst),
                                 "r"(smem_addr(ob)), "r"(static_cast<unsigned>(rec_tile * E))
                                 : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            } else {
                for (size_t i2 = static_cast<size_t>(et); i2 < static_cast<size_t>(rows) * p.NO; i2 += NE) gdst[i2] = ob[i2];
                named_bar_sync(1, NE);  // the staging buffer is read before the next tile overwrites it
            }
        }
        if (et == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(p.tmem_cols)
                     : "memory");
}

// CUDA-core kernel for the shapes and types the tensor-core kernel does not
// take: one warp per 4 pixels; for every output channel the lanes read the
// weight row and the 4 input rows (coalesced; both stay in L1/L2) and a warp
// reduction gives the 4 sums.
template <typename T>
__global__ void __launch_bounds__(256)
predictor_plain_kernel(const T* __restrict__ y, const T* __restrict__ w, const float* __restrict__ bias,
                       T* __restrict__ rec, PredParams p) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (long long m0 = (static_cast<long long>(blockIdx.x) * 8 + warp) * 4; m0 < p.M;
         m0 += static_cast<long long>(gridDim.x) * 32) {
        const int np = static_cast<int>(min(4LL, p.M - m0));
        const T* yr = y + m0 * p.C;
        for (int o = 0; o < p.NO; ++o) {
            const T* wr = w + static_cast<size_t>(o) * p.C;
            float a[4] = {0.f, 0.f, 0.f, 0.f};
            for (int c = lane; c < p.C; c += 32) {
                const float wv = ElemTraits<T>::to_float(__ldg(wr + c));
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (q < np) a[q] = fmaf(wv, ElemTraits<T>::to_float(__ldg(yr + static_cast<size_t>(q) * p.C + c)), a[q]);
            }
#pragma unroll
            for (int q = 0; q < 4; ++q)
                for (int off = 16; off > 0; off >>= 1) a[q] += __shfl_xor_sync(0xffffffffu, a[q], off);
            if (lane < np) {
                const float acc = (lane == 0 ? a[0] : lane == 1 ? a[1] : lane == 2 ? a[2] : a[3]) + (bias ? bias[o] : 0.f);
                T r;
                if constexpr (sizeof(T) == 4) r = acc;
                else r = from_float<T>(acc);
                rec[static_cast<size_t>(m0 + lane) * p.NO + pred_dest(o, p.G, p.P)] = r;
            }
        }
    }
}

}  // namespace dcnv4
