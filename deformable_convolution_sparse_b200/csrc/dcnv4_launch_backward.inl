// Launcher of the backward. Included by dcnv4.cu inside its anonymous
// namespace, after dcnv4_host_common.inl.
// Backward: grad_x is cleared on the stream, then one kernel computes every
// gradient. Vector path (4 channels per thread, float4 reductions) when the
// pointers and channel counts allow it, element path otherwise.
template <typename T>
int launch_backward(const void* x, const void* om, const void* go, float* gx, float* gom, float* gz, FwdParams p,
                    cudaStream_t stream) {
    constexpr int E = sizeof(T);
    const bool vec = aligned(x, 4 * E) && aligned(go, 4 * E) && aligned(gx, 16) && p.C % 4 == 0 && p.Cg % 4 == 0;
    const int cpl = vec ? 4 : 1;
    p.chunks = p.Cg / cpl;
    int lanes = 1;
    while (lanes < p.chunks && lanes < 32) lanes <<= 1;
    p.lanes = lanes;
    // units per block: full warps, records and fp32 gradient records in shared memory
    const size_t R = static_cast<size_t>(3) * p.npts;
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
        kernel<<<static_cast<unsigned>(blocks), threads, smem, stream>>>(xt, omt, got, gx, gom, gz, p);
        return launch_status();
    };
    const bool k3 = p.K == 3;
    // 16-channel groups on the vector path: four lanes of one chunk each, lanes known at compile time
    const bool four = vec && p.chunks == 4 && lanes == 4;
    if (p.flags != 0) {  // the variants: their own instantiations, so that the plain backward carries none of it
        if (four) return k3 ? run(dcnv4::bwd_kernel<T, 4, 3, true, 4>) : run(dcnv4::bwd_kernel<T, 4, 0, true, 4>);
        if (vec) return k3 ? run(dcnv4::bwd_kernel<T, 4, 3, true>) : run(dcnv4::bwd_kernel<T, 4, 0, true>);
        return k3 ? run(dcnv4::bwd_kernel<T, 1, 3, true>) : run(dcnv4::bwd_kernel<T, 1, 0, true>);
    }
    if (four) return k3 ? run(dcnv4::bwd_kernel<T, 4, 3, false, 4>) : run(dcnv4::bwd_kernel<T, 4, 0, false, 4>);
    if (vec) return k3 ? run(dcnv4::bwd_kernel<T, 4, 3, false>) : run(dcnv4::bwd_kernel<T, 4, 0, false>);
    return k3 ? run(dcnv4::bwd_kernel<T, 1, 3, false>) : run(dcnv4::bwd_kernel<T, 1, 0, false>);
}
