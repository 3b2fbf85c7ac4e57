// Interface between the translation units of libdcnv4.so (not installed, not
// part of the C ABI): the forward of each storage type is compiled in its own
// unit (dcnv4_fwd_f32.cu, dcnv4_fwd_f16.cu, dcnv4_fwd_bf16.cu) so that the
// kernel specialisations build in parallel; dcnv4.cu holds the C ABI.
#pragma once

#include <cuda_runtime.h>

#include "dcnv4_kernels.cuh"

// Returned by the forward launchers when a trace was asked for but the shape
// ran on the global-gather kernel, which has no tracing build (the output is
// written all the same).
#define DCNV4_NOT_TRACED 1000

namespace dcnv4_host {

// Launches the forward for x, offset_mask, out of one storage type. `status`:
// device address of the status word; `trace`: NULL, or device int4
// [units * points] for the ring kernel's tracing build.
int forward_f32(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status, int4* trace,
                cudaStream_t stream);
int forward_f16(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status, int4* trace,
                cudaStream_t stream);
int forward_bf16(const void* x, const void* om, void* out, const dcnv4::FwdParams& p, unsigned* status, int4* trace,
                 cudaStream_t stream);

// The forward's plan for a geometry on `nsm` SMs, without launching (15
// fields, the order of dcnv4_forward_plan in dcnv4.h).
int plan_f32(const dcnv4::FwdParams& p, int nsm, int* fields);
int plan_f16(const dcnv4::FwdParams& p, int nsm, int* fields);
int plan_bf16(const dcnv4::FwdParams& p, int nsm, int* fields);

}  // namespace dcnv4_host
