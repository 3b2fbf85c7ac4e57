// Forward aggregation, storage type __nv_bfloat16: the ring kernel, the global-gather
// fallback and their launcher (see dcnv4_launch_forward.inl).
#include "dcnv4_fwd_common.inl"

int dcnv4_host::forward_bf16(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status,
                          int4* trace, cudaStream_t stream) {
    return launch_forward<__nv_bfloat16>(x, om, out, p, status, trace, stream);
}

int dcnv4_host::plan_bf16(const dcnv4::FwdParams& p, int nsm, int* fields) {
    return plan_fields<__nv_bfloat16>(p, nsm, fields);
}
