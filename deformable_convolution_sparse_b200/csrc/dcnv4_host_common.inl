// Host-side helpers shared by the launchers of libdcnv4.so (argument checks,
// tensor-map encoding, device queries). Included by dcnv4.cu inside its
// anonymous namespace; not a stand-alone header.

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

constexpr int kThreads = 256;

constexpr size_t kTileSmemLimit = 226 * 1024;  // dynamic shared memory per CTA (sm_100: 227 KB with the static part)

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

// Raises a kernel's dynamic shared-memory limit, once per kernel and device
// (function attributes belong to each device's context); returns the result
// of that first call.
cudaError_t smem_limit_once(const void* kern, int bytes) {
    static std::mutex mu;
    static std::map<std::pair<const void*, int>, cudaError_t> done;
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_pair(kern, dev);
    if (auto it = done.find(key); it != done.end()) return it->second;
    const cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    done.emplace(key, r);
    return r;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 0;
    return n;
}
