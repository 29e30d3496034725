// dispatch.cu -- picks the kernel sequence for one validated mixer call.
#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

size_t workspace_bytes_for(const bimamba_dims &d)
{
    // one size serves both the scan and the cached decode of these dims
    size_t n = tc_path_supported(d) ? tc_workspace_bytes(d) : 0;
    if (decode_tc_supported(d)) n = n > decode_tc_workspace_bytes(d) ? n : decode_tc_workspace_bytes(d);
    return n;
}

cudaError_t launch_bimamba(const Problem &p, cudaStream_t stream)
{
    const bimamba_dims &d = p.dims;
    // bf16 at the model's head shape runs on the tensor cores; fp32 (which
    // needs a 1e-4 bound that bf16 operands cannot hold) and other head
    // shapes run on the sequential fp32 kernel.
    if (tc_path_supported(d)) return launch_ssd_tc(p, stream);
    if (d.dtype == BIMAMBA_F32) return launch_scan_seq<float>(p, stream);
    return launch_scan_seq<__nv_bfloat16>(p, stream);
}

}  // namespace bimamba
