// Host side of libdcnv4.so: argument checks, kernel selection and launch.
// The C ABI is declared (with the meaning of every argument) in include/dcnv4.h.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <array>
#include <cmath>
#include <map>
#include <mutex>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "dcnv4.h"
#include "dcnv4_async.cuh"
#include "dcnv4_internal.h"
#include "dcnv4_kernels.cuh"
#include "dcnv4_backward.cuh"
#include "dcnv4_predictor.cuh"

namespace dcnv4 {

// Device-side status word (kStatus* bits), read and cleared from the host
// through dcnv4_device_status(). The kernels of every translation unit get its
// device address as a parameter.
__device__ unsigned int g_device_status;

// Self-test of the bounded wait: arms an mbarrier for 16 bytes that never
// arrive (no copy is issued), waits `limit_ns`, records the timeout in
// *status and returns. Nothing is in flight, so nothing faults or hangs.
__global__ void selftest_wait_timeout_kernel(unsigned long long limit_ns, unsigned* status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
        mbar_expect_tx(&bar, 16);
        mbar_arrive(&bar);
        if (!mbar_wait_bounded(&bar, 0, limit_ns)) atomicOr(status, kStatusSelftestTimeout);
    }
}

// Shared-memory gather probe (dcnv4_probe_smem_gather): per CTA cycle counts.
constexpr int kProbeMaxCtas = 1024;
__device__ unsigned long long g_probe_cycles[kProbeMaxCtas];

// Every thread reads 16-byte chunks of 128-byte shared-memory rows picked by a
// per-thread linear congruential sequence (a power-of-two row count, so the
// pick is a mask), each lane of a quarter warp at a different 16-byte bank
// position: one 128-byte wavefront per quarter warp and load, whatever the
// rows. pattern 0: one chunk per pick; pattern 1: the forward's gather, 2x2
// corners x 2 chunks of a 128-byte pixel in a 26-pixel-wide window with the
// chunk rotation of the ring kernel (8 loads per pick).
__global__ void __launch_bounds__(512)
probe_smem_gather_kernel(int pattern, int iters) {
    extern __shared__ __align__(128) unsigned char psm[];
    constexpr int kRows = 512;  // 64 KB
    for (int i = threadIdx.x; i < kRows * 32; i += blockDim.x) reinterpret_cast<unsigned*>(psm)[i] = i * 2654435761u;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    unsigned s = 12345u + 977u * (blockIdx.x * blockDim.x + threadIdx.x);
    unsigned acc = 0;
    const unsigned long long t0 = clock64();
    if (pattern == 0) {
        for (int it = 0; it < iters; ++it) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                s = s * 1664525u + 1013904223u;
                const unsigned off = ((s >> 9) & (kRows - 1)) * 128u + (((lane & 7) + j) & 7) * 16u;
                const uint4 v = *reinterpret_cast<const uint4*>(psm + off);
                acc ^= v.x ^ v.y ^ v.z ^ v.w;
            }
        }
    } else {
        // window of 19 x 26 pixels of 128 bytes; corners of a pixel at (r, c): +128, +26*128
        const int gl = lane & 3, rot = (lane & 7) >> 2;
        for (int it = 0; it < iters; ++it) {
            s = s * 1664525u + 1013904223u;
            const unsigned r = (s >> 10) % 18u, c = (s >> 20) % 25u;
            const unsigned base = (r * 26u + c) * 128u + gl * 32u;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const unsigned pc = base + ((rot + j) & 1) * 16u;
                const uint4 a = *reinterpret_cast<const uint4*>(psm + pc);
                const uint4 b = *reinterpret_cast<const uint4*>(psm + pc + 128u);
                const uint4 c2 = *reinterpret_cast<const uint4*>(psm + pc + 26u * 128u);
                const uint4 d = *reinterpret_cast<const uint4*>(psm + pc + 27u * 128u);
                // every word of every load is used, so each stays one 16-byte load
                acc ^= a.x ^ a.y ^ a.z ^ a.w ^ b.x ^ b.y ^ b.z ^ b.w;
                acc ^= c2.x ^ c2.y ^ c2.z ^ c2.w ^ d.x ^ d.y ^ d.z ^ d.w;
            }
        }
    }
    const unsigned long long t1 = clock64();
    if (acc == 0x9e3779b9u) reinterpret_cast<unsigned*>(psm)[0] = acc;  // keeps the loads
    if (threadIdx.x == 0) g_probe_cycles[blockIdx.x] = t1 - t0;
}

// Shared-memory atomic probe (dcnv4_probe_red_shared): every thread adds 1 to
// a word of a 32 KB shared array, each lane of a warp on its own bank (the
// word a lane picks is lane + 32 * random row), as fp32 adds or as 32-bit
// integer adds. The rate decides whether a backward could accumulate grad_x
// contributions in shared memory before sending them to L2.
template <bool F32>
__global__ void __launch_bounds__(512) probe_red_shared_kernel(int iters, float* sink) {
    __shared__ float words[8192];
    for (int i = threadIdx.x; i < 8192; i += blockDim.x) words[i] = 0.f;
    __syncthreads();
    const unsigned lane = threadIdx.x & 31u;
    unsigned s = 12345u + 977u * threadIdx.x + 31u * blockIdx.x;
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
        s = s * 1664525u + 1013904223u;
        const unsigned idx = ((s >> 8) & 255u) * 32u + lane;
        if constexpr (F32) atomicAdd(&words[idx], 1.0f);
        else atomicAdd(reinterpret_cast<unsigned*>(&words[idx]), 1u);
    }
    __syncthreads();
    const unsigned long long t1 = clock64();
    if (threadIdx.x == 0) g_probe_cycles[blockIdx.x] = t1 - t0;
    if (threadIdx.x == 0 && words[7] == -1.f) sink[0] = words[7];  // keeps the adds
}

// Global reduction probe (dcnv4_probe_red_global): every warp issues 16-byte
// fp32 vector reductions (red.global.add.v4.f32) in groups of `group` lanes,
// each group covering one segment of group*16 contiguous bytes at a random
// segment of a buffer that stays in L2, 32/group segments per instruction.
// The rate bounds the backward's scatter into grad_x, whose lanes send each
// corner's group slice as such a segment.
__global__ void __launch_bounds__(512)
probe_red_global_kernel(float* buf, unsigned nseg_mask, int group, int iters) {
    const int lane = threadIdx.x & 31;
    const int gi = lane / group, gl = lane - gi * group;
    unsigned s = 0x9e3779b9u ^ (blockIdx.x * 7919u + (threadIdx.x >> 5) * 104729u);
    __syncthreads();
    const unsigned long long t0 = clock64();
    for (int it = 0; it < iters; ++it) {
        s = s * 1664525u + 1013904223u;
        unsigned r = s ^ (static_cast<unsigned>(gi) * 2654435761u);  // the group's own segment
        r ^= r >> 13;
        r *= 0x5bd1e995u;
        r ^= r >> 15;
        float* q = buf + static_cast<size_t>(r & nseg_mask) * group * 4 + gl * 4;
        atomicAdd(reinterpret_cast<float4*>(q), make_float4(1.f, 1.f, 1.f, 1.f));
    }
    __syncthreads();
    const unsigned long long t1 = clock64();
    if (threadIdx.x == 0) g_probe_cycles[blockIdx.x] = t1 - t0;
}

}  // namespace dcnv4

namespace {

using dcnv4::FwdParams;

#include "dcnv4_host_common.inl"

#include "dcnv4_launch_backward.inl"

#include "dcnv4_launch_predictor.inl"

constexpr int kMaxDevices = 64;

// Device address of the status word on the current device, looked up once per
// device (cudaGetSymbolAddress with that device current); NULL on failure.
unsigned* status_word() {
    static unsigned* addr[kMaxDevices];
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, dcnv4::g_device_status) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<unsigned*>(p);
    }
    return addr[dev];
}

// Three non-blocking streams per device for the host-memory entry points,
// created on first use and kept for the life of the process.
struct HostPipe {
    cudaStream_t s[3] = {nullptr, nullptr, nullptr};
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
        for (int i = 0; i < 3; ++i)
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
    p.Hout = Hout; p.Wout = Wout; p.row0 = 0;
    p.units = N * Hout * Wout * G;
    p.offset_scale = offset_scale;
    p.flags = static_cast<int>(flags);
    const bool rc = (flags & DCNV4_FLAG_REMOVE_CENTER) != 0u;
    p.npts = p.KK - (rc ? 1 : 0);
    p.kc = rc ? (p.KK - 1) / 2 : p.KK;
    p.center_logit = center_logit;
    return p;
}

// The forward of one storage type through its translation unit.
int run_forward(const void* x, const void* om, void* out, const FwdParams& p, int dtype, int4* trace,
                cudaStream_t s) {
    unsigned* status = status_word();
    if (!status) return DCNV4_ERR_CUDA;
    switch (dtype) {
        case DCNV4_F32: return dcnv4_host::forward_f32(x, om, out, p, status, trace, s);
        case DCNV4_F16: return dcnv4_host::forward_f16(x, om, out, p, status, trace, s);
        default: return dcnv4_host::forward_bf16(x, om, out, p, status, trace, s);
    }
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
    return run_forward(x, offset_mask, out, p, dtype, nullptr, static_cast<cudaStream_t>(stream));
}

int dcnv4_forward_plan(int N, int H, int W, int C, int G, int K, int stride, int pad, int dilation, int dtype,
                       unsigned flags, int nsm, int* fields, int nfields) {
    long long nx = 0, nout = 0, nom = 0;
    int rc = check_sizes(N, H, W, C, G, K, stride, pad, dilation, 1.0f, dtype, &nx, &nout, &nom);
    if (rc) return rc;
    if (flags & ~static_cast<unsigned>(DCNV4_FLAG_SOFTMAX | DCNV4_FLAG_REMOVE_CENTER | DCNV4_FLAG_CENTER_SCALE))
        return DCNV4_ERR_FLAGS;
    if ((flags & DCNV4_FLAG_REMOVE_CENTER) && (K % 2 == 0 || K < 3)) return DCNV4_ERR_SHAPE;
    if (!fields) return DCNV4_ERR_NULL;
    if (nfields < DCNV4_PLAN_FIELDS || nsm < 1 || nsm > 1024) return DCNV4_ERR_SHAPE;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const FwdParams p = make_params(N, H, W, C, G, K, stride, pad, dilation, 1.0f, Hout, Wout, flags);
    switch (dtype) {
        case DCNV4_F32: return dcnv4_host::plan_f32(p, nsm, fields);
        case DCNV4_F16: return dcnv4_host::plan_f16(p, nsm, fields);
        default: return dcnv4_host::plan_bf16(p, nsm, fields);
    }
}

int dcnv4_forward(const void* x, const void* offset_mask, void* out,
                  int N, int H, int W, int C, int G, int K,
                  int stride, int pad, int dilation, float offset_scale, int dtype,
                  void* stream) {
    return dcnv4_forward_ex(x, offset_mask, nullptr, out, N, H, W, C, G, K, stride, pad, dilation, offset_scale,
                            dtype, 0u, stream);
}

int dcnv4_forward_trace(const void* x, const void* offset_mask, void* out, int32_t* trace,
                        int N, int H, int W, int C, int G, int K,
                        int stride, int pad, int dilation, float offset_scale, int dtype,
                        void* stream) {
    const int rc = dcnv4_validate(x, offset_mask, out, N, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype);
    if (rc) return rc;
    if (N == 0) return DCNV4_OK;
    if (!trace) return DCNV4_ERR_NULL;
    if (!aligned(trace, 16)) return DCNV4_ERR_ALIGN;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const int e = elem_size(dtype);
    const long long npts = static_cast<long long>(N) * Hout * Wout * G * K * K;
    if (4 * npts >= kLimit) return DCNV4_ERR_TOO_LARGE;
    const long long nx = static_cast<long long>(N) * H * W * C, nout = static_cast<long long>(N) * Hout * Wout * C;
    if (overlap(trace, 16 * npts, x, nx * e) || overlap(trace, 16 * npts, offset_mask, 3 * npts * e) ||
        overlap(trace, 16 * npts, out, nout * e))
        return DCNV4_ERR_ALIAS;
    const FwdParams p = make_params(N, H, W, C, G, K, stride, pad, dilation, offset_scale, Hout, Wout);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int4* tr = reinterpret_cast<int4*>(trace);
    const int frc = run_forward(x, offset_mask, out, p, dtype, tr, s);
    if (frc != DCNV4_NOT_TRACED) return frc;
    // the global-gather kernel ran: trace its sampling with the code it shares
    const long long want = (npts + 255) / 256;
    const unsigned blocks = static_cast<unsigned>(want < 148 * 32 ? want : 148 * 32);
    switch (dtype) {
        case DCNV4_F32:
            dcnv4::trace_index_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(offset_mask), tr, p);
            break;
        case DCNV4_F16:
            dcnv4::trace_index_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(offset_mask), tr, p);
            break;
        default:
            dcnv4::trace_index_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
                static_cast<const __nv_bfloat16*>(offset_mask), tr, p);
            break;
    }
    return launch_status();
}

int dcnv4_backward_ex(const void* x, const void* offset_mask, const void* center_logit, const void* grad_out,
                      float* grad_x, float* grad_offset_mask, float* grad_center_logit,
                      int N, int H, int W, int C, int G, int K,
                      int stride, int pad, int dilation, float offset_scale, int dtype, unsigned flags,
                      void* stream) {
    long long nx = 0, nout = 0, nom = 0;
    int rc = check_sizes(N, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype, &nx, &nout, &nom);
    if (rc) return rc;
    if (flags & ~static_cast<unsigned>(DCNV4_FLAG_SOFTMAX | DCNV4_FLAG_REMOVE_CENTER | DCNV4_FLAG_CENTER_SCALE))
        return DCNV4_ERR_FLAGS;
    if ((flags & DCNV4_FLAG_REMOVE_CENTER) && (K % 2 == 0 || K < 3)) return DCNV4_ERR_SHAPE;
    nom = nom / (3LL * K * K) * 3LL * points_per_unit(K, flags);
    const long long ngate = nout / C * G;
    const bool cs = (flags & DCNV4_FLAG_CENTER_SCALE) != 0u;
    if (N == 0) return DCNV4_OK;
    if (!x || !offset_mask || !grad_out || !grad_x || !grad_offset_mask) return DCNV4_ERR_NULL;
    if (cs && (!center_logit || !grad_center_logit)) return DCNV4_ERR_NULL;
    const int e = elem_size(dtype);
    if (!aligned(x, e) || !aligned(offset_mask, e) || !aligned(grad_out, e) || !aligned(grad_x, 4) ||
        !aligned(grad_offset_mask, 4) || (cs && (!aligned(center_logit, e) || !aligned(grad_center_logit, 4))))
        return DCNV4_ERR_ALIGN;
    const void* inputs[4] = {x, offset_mask, grad_out, cs ? center_logit : nullptr};
    const long long in_bytes[4] = {nx * e, nom * e, nout * e, cs ? ngate * e : 0};
    for (int i = 0; i < 4; ++i)
        if (overlap(grad_x, nx * 4, inputs[i], in_bytes[i]) || overlap(grad_offset_mask, nom * 4, inputs[i], in_bytes[i]) ||
            (cs && overlap(grad_center_logit, ngate * 4, inputs[i], in_bytes[i])))
            return DCNV4_ERR_ALIAS;
    if (overlap(grad_x, nx * 4, grad_offset_mask, nom * 4) ||
        (cs && (overlap(grad_center_logit, ngate * 4, grad_x, nx * 4) ||
                overlap(grad_center_logit, ngate * 4, grad_offset_mask, nom * 4))))
        return DCNV4_ERR_ALIAS;
    int Hout = 0, Wout = 0;
    dcnv4_output_shape(H, W, K, stride, pad, dilation, &Hout, &Wout);
    const FwdParams p = make_params(N, H, W, C, G, K, stride, pad, dilation, offset_scale, Hout, Wout, flags,
                                    cs ? center_logit : nullptr);
    float* gz = cs ? grad_center_logit : nullptr;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32: return launch_backward<float>(x, offset_mask, grad_out, grad_x, grad_offset_mask, gz, p, s);
        case DCNV4_F16: return launch_backward<__half>(x, offset_mask, grad_out, grad_x, grad_offset_mask, gz, p, s);
        default: return launch_backward<__nv_bfloat16>(x, offset_mask, grad_out, grad_x, grad_offset_mask, gz, p, s);
    }
}

int dcnv4_backward(const void* x, const void* offset_mask, const void* grad_out,
                   float* grad_x, float* grad_offset_mask,
                   int N, int H, int W, int C, int G, int K,
                   int stride, int pad, int dilation, float offset_scale, int dtype,
                   void* stream) {
    return dcnv4_backward_ex(x, offset_mask, nullptr, grad_out, grad_x, grad_offset_mask, nullptr, N, H, W, C, G, K,
                             stride, pad, dilation, offset_scale, dtype, 0u, stream);
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
    p.status = status_word();
    if (!p.status) return DCNV4_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    switch (dtype) {
        case DCNV4_F32: return launch_predictor<float>(y, weight, bias, offset_mask, p, s);
        case DCNV4_F16: return launch_predictor<__half>(y, weight, bias, offset_mask, p, s);
        default: return launch_predictor<__nv_bfloat16>(y, weight, bias, offset_mask, p, s);
    }
}

namespace {

// The forward's plan (dcnv4_forward_plan's fields) for the geometry in p on this device.
int plan_of(const FwdParams& p, int dtype, int* fields) {
    const int nsm = sm_count();
    if (nsm <= 0) return DCNV4_ERR_CUDA;
    switch (dtype) {
        case DCNV4_F32: return dcnv4_host::plan_f32(p, nsm, fields);
        case DCNV4_F16: return dcnv4_host::plan_f16(p, nsm, fields);
        default: return dcnv4_host::plan_bf16(p, nsm, fields);
    }
}

// True when every band of `bands` equal row ranges runs the kernel, window kind and halo of the
// whole image, which makes its outputs the whole-image launch's bit for bit (the planner takes
// the halo and window kind from the image geometry; the rest of a plan leaves each sample's
// arithmetic unchanged). A band whose plan would fall back to another kernel is not used.
// Kept per geometry, band count, storage type and device: a few plan look-ups (string keys
// built from the planner's environment switches) would otherwise cost tens of microseconds of
// host time on every call. Not kept while a planner override is set (tuning runs may change it
// between calls).
bool bands_match_image(int N, int H, int W, int C, int G, int K, int stride, int pad, int dilation, int Hout,
                       int Wout, int dtype, int bands) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    static std::mutex mu;
    static std::map<std::array<int, 12>, bool> cache;
    bool keep = true;
    for (const char* e : {"DCNV4_HALO", "DCNV4_WINDOW", "DCNV4_TILE", "DCNV4_GS", "DCNV4_NREC", "DCNV4_RING"})
        if (std::getenv(e)) keep = false;
    const std::array<int, 12> key = {N, H, W, C, G, K, stride, pad, dilation, dtype, bands, dev};
    if (keep) {
        std::lock_guard<std::mutex> lock(mu);
        if (auto it = cache.find(key); it != cache.end()) return it->second;
    }
    bool match = true;
    int whole[DCNV4_PLAN_FIELDS], part[DCNV4_PLAN_FIELDS];
    if (plan_of(make_params(N, H, W, C, G, K, stride, pad, dilation, 1.0f, Hout, Wout), dtype, whole)) match = false;
    for (int b = 0; b < bands && match; ++b) {
        const int rows = static_cast<int>((static_cast<long long>(Hout) * (b + 1)) / bands) -
                         static_cast<int>((static_cast<long long>(Hout) * b) / bands);
        if (plan_of(make_params(1, H, W, C, G, K, stride, pad, dilation, 1.0f, rows, Wout), dtype, part)) {
            match = false;
            break;
        }
        for (int i = 0; i < 3; ++i)  // kernel, window kind, halo
            if (part[i] != whole[i]) match = false;
    }
    if (keep) {
        std::lock_guard<std::mutex> lock(mu);
        if (cache.size() >= 256) cache.clear();
        cache.emplace(key, match);
    }
    return match;
}

}  // namespace

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
    // The library's three streams have one role each: s[0] copies the inputs in, s[1] runs the
    // kernels, s[2] copies the results out. A chunk's kernel waits for its own inputs (ev_in) and
    // its copy out for its kernel (ev_k); the copies in wait for nothing but each other, so the
    // host-to-device direction, which carries x and offset_mask against the other's one result,
    // runs back to back while the other overlaps it. cudaStreamWaitEvent takes the event's latest
    // record at the time of the call, so one event per role serves every chunk.
    cudaEvent_t ev_start = nullptr, ev_in = nullptr, ev_k = nullptr, ev_done[3] = {nullptr, nullptr, nullptr};
    bool queued = false;  // copies or kernels are on the library's streams
    // Ends the call: once anything is queued the caller's stream waits for all
    // of it, on success and after an error alike, so that no copy into out_host
    // is still pending when the caller's stream moves on.
    auto fail = [&](int code) {
        if (queued) {
            for (int i = 0; i < 3; ++i) {
                const bool ok = ev_done[i] && cudaEventRecord(ev_done[i], pipe->s[i]) == cudaSuccess &&
                                cudaStreamWaitEvent(user, ev_done[i], 0) == cudaSuccess;
                if (!ok && code == DCNV4_OK) code = DCNV4_ERR_CUDA;
            }
        }
        // events may be destroyed while pending: the waits already queued keep their meaning
        for (cudaEvent_t ev : {ev_start, ev_in, ev_k, ev_done[0], ev_done[1], ev_done[2]})
            if (ev) cudaEventDestroy(ev);
        return code;
    };
    for (cudaEvent_t* ev : {&ev_start, &ev_in, &ev_k, &ev_done[0], &ev_done[1], &ev_done[2]})
        if (cudaEventCreateWithFlags(ev, cudaEventDisableTiming) != cudaSuccess) return fail(DCNV4_ERR_CUDA);
    if (cudaEventRecord(ev_start, user) != cudaSuccess) return fail(DCNV4_ERR_CUDA);
    for (int i = 0; i < 3; ++i)
        if (cudaStreamWaitEvent(pipe->s[i], ev_start, 0) != cudaSuccess) return fail(DCNV4_ERR_CUDA);

    // Chunks of about 8 MiB of input copies each, 2 to 8 of them: every copy costs the copy
    // engine a few microseconds beyond its bytes (measured ~3.7 us on PCIe 5), while the last
    // chunk's kernel and copy out are the part of the call that nothing overlaps, so neither many
    // small chunks nor one large one. DCNV4_HOST_CHUNKS sets the count (tuning runs). A chunk is
    // whole images; with fewer images than chunks each image is cut into bands of output rows
    // instead, each band a launch over its rows of the whole image (FwdParams::row0), so that the
    // last launch and copy out stay short for a batch of a few large images.
    // When a result is no larger than an image's offset_mask records, x goes over first in one
    // copy and only the records are chunked: one copy less per chunk, and the results' copies
    // out still have the records' transfer time to overlap with (with larger results they would
    // queue up behind the last chunk).
    const size_t in_bytes = static_cast<size_t>(N) * (x_img + om_img);
    int chunks = static_cast<int>(std::min<size_t>(8, std::max<size_t>(2, in_bytes >> 23)));
    if (const char* c = std::getenv("DCNV4_HOST_CHUNKS")) chunks = std::max(1, std::atoi(c));
    const bool x_first = out_img <= om_img;
    const char* xh = static_cast<const char*>(x_host);
    const char* omh = static_cast<const char*>(offset_mask_host);
    char* oh = static_cast<char*>(out_host);
    char* xd = static_cast<char*>(x_dev);
    char* omd = static_cast<char*>(offset_mask_dev);
    char* od = static_cast<char*>(out_dev);
    cudaStream_t s_in = pipe->s[0], s_k = pipe->s[1], s_out = pipe->s[2];
    if (x_first) {  // queued first, so the copy runs while the pieces are worked out
        queued = true;
        if (cudaMemcpyAsync(xd, xh, N * x_img, cudaMemcpyHostToDevice, s_in) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
    }
    int bands = chunks > N ? std::min(Hout, (chunks + N - 1) / N) : 1;  // pieces per image
    if (bands > 1 && !bands_match_image(N, H, W, C, G, K, stride, pad, dilation, Hout, Wout, dtype, bands))
        bands = 1;
    const int pieces = bands > 1 ? N * bands : std::min(chunks, N);
    const size_t om_row = om_img / Hout, out_row = out_img / Hout;  // bytes per output row
    for (int c = 0; c < pieces; ++c) {
        // piece c: images [n0, n1), output rows [r0, r1) of each (all rows unless cut into bands)
        int n0, n1, r0 = 0, r1 = Hout;
        if (bands > 1) {
            n0 = c / bands;
            n1 = n0 + 1;
            const int b = c - n0 * bands;
            r0 = static_cast<int>((static_cast<long long>(Hout) * b) / bands);
            r1 = static_cast<int>((static_cast<long long>(Hout) * (b + 1)) / bands);
        } else {
            n0 = static_cast<int>((static_cast<long long>(N) * c) / pieces);
            n1 = static_cast<int>((static_cast<long long>(N) * (c + 1)) / pieces);
        }
        const int nc = n1 - n0;
        if (nc == 0 || r1 == r0) continue;
        queued = true;
        const size_t om_off = n0 * om_img + r0 * om_row, om_len = bands > 1 ? (r1 - r0) * om_row : nc * om_img;
        const size_t out_off = n0 * out_img + r0 * out_row, out_len = bands > 1 ? (r1 - r0) * out_row : nc * out_img;
        if ((!x_first && r0 == 0 &&
             cudaMemcpyAsync(xd + n0 * x_img, xh + n0 * x_img, nc * x_img, cudaMemcpyHostToDevice, s_in) !=
                 cudaSuccess) ||
            cudaMemcpyAsync(omd + om_off, omh + om_off, om_len, cudaMemcpyHostToDevice, s_in) != cudaSuccess ||
            cudaEventRecord(ev_in, s_in) != cudaSuccess || cudaStreamWaitEvent(s_k, ev_in, 0) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
        if (bands > 1) {
            FwdParams p = make_params(1, H, W, C, G, K, stride, pad, dilation, offset_scale, r1 - r0, Wout);
            p.row0 = r0;
            rc = run_forward(xd + n0 * x_img, omd + om_off, od + out_off, p, dtype, nullptr, s_k);
        } else {
            rc = dcnv4_forward(xd + n0 * x_img, omd + om_off, od + out_off, nc, H, W, C, G, K, stride, pad, dilation,
                               offset_scale, dtype, s_k);
        }
        if (rc) return fail(rc);
        if (cudaEventRecord(ev_k, s_k) != cudaSuccess || cudaStreamWaitEvent(s_out, ev_k, 0) != cudaSuccess ||
            cudaMemcpyAsync(oh + out_off, od + out_off, out_len, cudaMemcpyDeviceToHost, s_out) != cudaSuccess)
            return fail(DCNV4_ERR_CUDA);
    }
    return fail(DCNV4_OK);
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
    unsigned* status = status_word();
    if (!status) return DCNV4_ERR_CUDA;
    dcnv4::selftest_wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status);
    return launch_status();
}

int dcnv4_probe_smem_gather(int pattern, double* bytes_per_clock_per_sm) {
    if (!bytes_per_clock_per_sm) return DCNV4_ERR_NULL;
    if (pattern != 0 && pattern != 1) return DCNV4_ERR_SHAPE;
    const int nsm = sm_count();
    if (nsm <= 0 || nsm > dcnv4::kProbeMaxCtas) return DCNV4_ERR_CUDA;
    constexpr int threads = 512, iters = 2048;
    const size_t smem = 512 * 128;
    if (cudaFuncSetAttribute(dcnv4::probe_smem_gather_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
        return DCNV4_ERR_CUDA;
    unsigned long long cyc[dcnv4::kProbeMaxCtas];
    for (int rep = 0; rep < 2; ++rep) {  // the first launch warms up
        dcnv4::probe_smem_gather_kernel<<<nsm, threads, smem>>>(pattern, iters);
        if (cudaGetLastError() != cudaSuccess) return DCNV4_ERR_LAUNCH;
        if (cudaDeviceSynchronize() != cudaSuccess) return DCNV4_ERR_CUDA;
    }
    if (cudaMemcpyFromSymbol(cyc, dcnv4::g_probe_cycles, sizeof(unsigned long long) * nsm) != cudaSuccess)
        return DCNV4_ERR_CUDA;
    unsigned long long mx = 1;
    for (int i = 0; i < nsm; ++i) mx = std::max(mx, cyc[i]);
    const double loads = static_cast<double>(threads) * iters * 8.0;  // 16-byte loads per CTA
    *bytes_per_clock_per_sm = loads * 16.0 / static_cast<double>(mx);
    return DCNV4_OK;
}

int dcnv4_probe_red_global(int segment_bytes, double* bytes_per_clock_per_sm) {
    if (!bytes_per_clock_per_sm) return DCNV4_ERR_NULL;
    if (segment_bytes != 32 && segment_bytes != 64 && segment_bytes != 128) return DCNV4_ERR_SHAPE;
    const int nsm = sm_count();
    if (nsm <= 0 || nsm > dcnv4::kProbeMaxCtas) return DCNV4_ERR_CUDA;
    constexpr int threads = 512, iters = 2000;
    constexpr size_t bytes = size_t{32} << 20;  // 32 MB: resident in L2
    const int group = segment_bytes / 16;
    const unsigned nseg = static_cast<unsigned>(bytes / static_cast<size_t>(segment_bytes));  // a power of two
    float* buf = nullptr;
    if (cudaMalloc(&buf, bytes) != cudaSuccess) return DCNV4_ERR_CUDA;
    int rc = DCNV4_OK;
    if (cudaMemset(buf, 0, bytes) != cudaSuccess) rc = DCNV4_ERR_CUDA;
    for (int rep = 0; rep < 2 && rc == DCNV4_OK; ++rep) {  // the first launch warms up
        dcnv4::probe_red_global_kernel<<<nsm, threads>>>(buf, nseg - 1, group, iters);
        if (cudaGetLastError() != cudaSuccess) rc = DCNV4_ERR_LAUNCH;
        else if (cudaDeviceSynchronize() != cudaSuccess) rc = DCNV4_ERR_CUDA;
    }
    unsigned long long cyc[dcnv4::kProbeMaxCtas];
    if (rc == DCNV4_OK &&
        cudaMemcpyFromSymbol(cyc, dcnv4::g_probe_cycles, sizeof(unsigned long long) * nsm) != cudaSuccess)
        rc = DCNV4_ERR_CUDA;
    if (cudaFree(buf) != cudaSuccess && rc == DCNV4_OK) rc = DCNV4_ERR_CUDA;
    if (rc != DCNV4_OK) return rc;
    unsigned long long mx = 1;
    for (int i = 0; i < nsm; ++i) mx = std::max(mx, cyc[i]);
    const double payload = static_cast<double>(threads) * iters * 16.0;  // bytes per CTA
    *bytes_per_clock_per_sm = payload / static_cast<double>(mx);
    return DCNV4_OK;
}

int dcnv4_probe_red_shared(int fp32, double* adds_per_clock_per_sm) {
    if (!adds_per_clock_per_sm) return DCNV4_ERR_NULL;
    if (fp32 != 0 && fp32 != 1) return DCNV4_ERR_SHAPE;
    const int nsm = sm_count();
    if (nsm <= 0 || nsm > dcnv4::kProbeMaxCtas) return DCNV4_ERR_CUDA;
    constexpr int threads = 512, iters = 4096;
    float* sink = nullptr;
    if (cudaMalloc(&sink, 16) != cudaSuccess) return DCNV4_ERR_CUDA;
    int rc = DCNV4_OK;
    for (int rep = 0; rep < 2 && rc == DCNV4_OK; ++rep) {  // the first launch warms up
        if (fp32) dcnv4::probe_red_shared_kernel<true><<<nsm, threads>>>(iters, sink);
        else dcnv4::probe_red_shared_kernel<false><<<nsm, threads>>>(iters, sink);
        if (cudaGetLastError() != cudaSuccess) rc = DCNV4_ERR_LAUNCH;
        else if (cudaDeviceSynchronize() != cudaSuccess) rc = DCNV4_ERR_CUDA;
    }
    unsigned long long cyc[dcnv4::kProbeMaxCtas];
    if (rc == DCNV4_OK &&
        cudaMemcpyFromSymbol(cyc, dcnv4::g_probe_cycles, sizeof(unsigned long long) * nsm) != cudaSuccess)
        rc = DCNV4_ERR_CUDA;
    if (cudaFree(sink) != cudaSuccess && rc == DCNV4_OK) rc = DCNV4_ERR_CUDA;
    if (rc != DCNV4_OK) return rc;
    unsigned long long mx = 1;
    for (int i = 0; i < nsm; ++i) mx = std::max(mx, cyc[i]);
    *adds_per_clock_per_sm = static_cast<double>(threads) * iters / static_cast<double>(mx);
    return DCNV4_OK;
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
    bool queued = false;  // copies or kernels are on the library's streams
    // Ends the call: once anything is queued the caller's stream waits for all
    // of it, on success and after an error alike (see dcnv4_forward_host).
    auto release = [&](int code) {
        if (queued) {
            for (int i = 0; i < 2; ++i) {
                const bool ok = ev_done[i] && cudaEventRecord(ev_done[i], pipe->s[i]) == cudaSuccess &&
                                cudaStreamWaitEvent(user, ev_done[i], 0) == cudaSuccess;
                if (!ok && code == DCNV4_OK) code = DCNV4_ERR_CUDA;
            }
        }
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
        queued = true;
        if (cudaMemcpyAsync(xd, xh + n0 * x_img, nc * x_img, cudaMemcpyHostToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(omd, omh + n0 * om_img, nc * om_img, cudaMemcpyHostToDevice, s) != cudaSuccess)
            return release(DCNV4_ERR_CUDA);
        rc = dcnv4_forward(xd, omd, od, nc, H, W, C, G, K, stride, pad, dilation, offset_scale, dtype, s);
        if (rc) return release(rc);
        if (cudaMemcpyAsync(oh + n0 * out_img, od, nc * out_img, cudaMemcpyDeviceToHost, s) != cudaSuccess)
            return release(DCNV4_ERR_CUDA);
    }
    return release(DCNV4_OK);
}
