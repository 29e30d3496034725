// noalloc.cu -- cached block decode for callers that cannot allocate device
// memory.
//
// bimamba_block_decode takes a caller-allocated workspace.  Some callers
// cannot provide one: a serving process whose memory pool has already
// reserved the whole device (a cudaMalloc from the library would fail or
// fight that pool), or a decode loop whose rules forbid any allocation once
// it is serving.  bimamba_block_decode_noalloc gives them the same operation
// with the scratch taken from a fixed array that lives in this library's own
// device memory.
//
// The array is a file-scope __device__ array of kScratchBytes; every GPU that
// loads the library holds it until the process exits.  Host code only sees
// a host-side stand-in for the array's name, so its device address is looked
// up once per device with cudaGetSymbolAddress (with that device current)
// and passed on as the workspace pointer.
#include <mutex>

#include "common.cuh"
#include "dispatch.h"

namespace bimamba {
namespace {

constexpr size_t kScratchBytes = 16u << 20;  // 16 MiB per device
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of this device's scratch array, resolved on first use.
void *scratch_address(int *status)
{
    static std::mutex mu;
    static void *addr[kMaxDevices] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = BIMAMBA_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
            *status = BIMAMBA_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    *status = BIMAMBA_OK;
    return addr[dev];
}

}  // namespace
}  // namespace bimamba

using namespace bimamba;

extern "C" {

size_t bimamba_noalloc_scratch_bytes(void) { return kScratchBytes; }

int bimamba_block_decode_noalloc(const bimamba_dims *d, const void *xbc_block,
                                 const void *dt_block, const float *A, const float *D,
                                 const float *conv_w, const float *conv_b, const float *state,
                                 const void *tail, void *y, float *state_out, void *tail_out,
                                 bimamba_stream_t stream)
{
    // the same argument checks as bimamba_block_decode, before anything is
    // queued on the stream: a rejected call launches nothing
    int st = check_block_decode(d, xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y,
                                state_out, tail_out);
    if (st != BIMAMBA_OK) return st;
    if (d->batch == 0) return BIMAMBA_OK;
    const size_t need = bimamba_workspace_bytes(d);
    if (need > kScratchBytes) return BIMAMBA_ERR_WORKSPACE;   // beyond the fixed scratch
    void *scratch = scratch_address(&st);
    if (st != BIMAMBA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // The decode kernels expect the scratch's meeting counters at zero.
    // Every call shares this array, so clear them (a previous call that
    // stopped early, e.g. on a timeout, could have left counters set); the
    // rest of the scratch is rewritten by every call.
    const size_t counters = tc_path_supported(*d) ? tc_counter_bytes(*d) : 0;
    if (counters > 0 && cudaMemsetAsync(scratch, 0, counters, s) != cudaSuccess)
        return BIMAMBA_ERR_CUDA;
    return bimamba_block_decode(d, xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y,
                                state_out, tail_out, scratch, kScratchBytes, stream);
}

}  // extern "C"
