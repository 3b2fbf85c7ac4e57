// Forward aggregation, storage type __half: the ring kernel, the global-gather
// fallback and their launcher (see dcnv4_launch_forward.inl).
#include "dcnv4_fwd_common.inl"

int dcnv4_host::forward_f16(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status,
                          int4* trace, cudaStream_t stream) {
    return launch_forward<__half>(x, om, out, p, status, trace, stream);
}

int dcnv4_host::plan_f16(const dcnv4::FwdParams& p, int nsm, int* fields) {
    return plan_fields<__half>(p, nsm, fields);
}
