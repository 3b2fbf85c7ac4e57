// Forward aggregation, storage type float: the ring kernel, the global-gather
// fallback and their launcher (see dcnv4_launch_forward.inl).
#include "dcnv4_fwd_common.inl"

int dcnv4_host::forward_f32(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status,
                          int4* trace, cudaStream_t stream) {
    return launch_forward<float>(x, om, out, p, status, trace, stream);
}

int dcnv4_host::plan_f32(const dcnv4::FwdParams& p, int nsm, int* fields) {
    return plan_fields<float>(p, nsm, fields);
}
