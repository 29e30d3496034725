// dispatch.cu -- picks the kernel sequence for one validated mixer call.
#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

size_t workspace_bytes_for(const bimamba_dims &d)
{
    (void)d;
    return 0;
}

cudaError_t launch_bimamba(const Problem &p, cudaStream_t stream)
{
    const bimamba_dims &d = p.dims;
    if (d.dtype == BIMAMBA_F32)
        return launch_scan_seq<float>(p.xbc, p.dt, p.A, p.D, p.conv_w, p.conv_b, p.tail, p.init,
                                      p.fin, p.y, d.batch, d.len, d.heads, d.headdim, d.d_state,
                                      stream);
    return launch_scan_seq<__nv_bfloat16>(p.xbc, p.dt, p.A, p.D, p.conv_w, p.conv_b, p.tail,
                                          p.init, p.fin, p.y, d.batch, d.len, d.heads, d.headdim,
                                          d.d_state, stream);
}

}  // namespace bimamba
