// Common part of the per-storage-type forward units (dcnv4_fwd_*.cu): the
// kernels, the host helpers and the launcher, all with internal linkage.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "dcnv4.h"
#include "dcnv4_internal.h"
#include "dcnv4_kernels.cuh"
#include "dcnv4_window.cuh"

namespace {

using dcnv4::FwdParams;

#include "dcnv4_host_common.inl"

#include "dcnv4_launch_forward.inl"

// The forward's plan for a geometry, without launching anything
// (dcnv4_forward_plan): the ring kernel's eligibility as in plan_ring (the
// pointers taken as 16-byte aligned) and its shape; field order in dcnv4.h.
template <typename T>
int plan_fields(const FwdParams& f, int nsm, int* out) {
    constexpr int E = sizeof(T);
    for (int i = 0; i < 15; ++i) out[i] = 0;
    out[0] = 1;  // the global-gather kernel unless the ring kernel takes the shape
    const int row_bytes = f.Cg * E;
    if ((f.C * E) % 16 || row_bytes % 16) return DCNV4_OK;
    const int Q = row_bytes / 16;
    if (!(Q == 1 || Q == 2 || Q == 4 || Q == 5 || Q == 8) || f.KK > 64) return DCNV4_OK;
    const RingShape sh = cached_ring_shape<T>(f, nsm);
    if (sh.score < 0.0) return DCNV4_OK;
    const int fields[15] = {0, sh.img, sh.R, sh.GS, sh.TW, sh.TH, sh.NR, sh.nrec, sh.units, sh.threads,
                            static_cast<int>(sh.smem), sh.UH, sh.UW, sh.WW, sh.GS * row_bytes};
    for (int i = 0; i < 15; ++i) out[i] = fields[i];
    return DCNV4_OK;
}

}  // namespace
