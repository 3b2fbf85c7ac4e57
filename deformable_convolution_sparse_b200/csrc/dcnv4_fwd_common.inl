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

}  // namespace
