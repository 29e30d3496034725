// common.cuh -- small device helpers shared by the sm_100a kernels of the
// bidirectional Mamba-2 mixer library.  Nothing here is shared with the CPU
// oracle.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bimamba.h"

namespace bimamba {

// Kernels that can detect an error at run time (a bounded wait that gave up)
// OR a bit into the per-device status word whose address the host passes
// them; bimamba_get_error reads and clears it.
enum : int { kStatusTimeout = 1, kStatusBadSlot = 2 };

__device__ __forceinline__ void record_error(int *status, int bit) {
    if (status) atomicOr(status, bit);
}

// Address of this device's status word (host side; defined in api.cu).
int *device_status_word();

// Host-side count of kernels this library has launched (defined in api.cu).
void count_launch(int n = 1);

// Caller-provided timing events around the main scan kernel (or null); see
// bimamba_set_timing_events.
struct TimingEvents {
    cudaEvent_t start;
    cudaEvent_t stop;
};
TimingEvents timing_events();

// ---- element loads / stores in the activation dtype -------------------------
template <typename T> struct Elem;

template <> struct Elem<float> {
    static __device__ __forceinline__ float load(const float *p) { return *p; }
    static __device__ __forceinline__ void store(float *p, float v) { *p = v; }
};

template <> struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16 *p) {
        return __bfloat162float(*p);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, float v) {
        *p = __float2bfloat16_rn(v);
    }
};

// 8 consecutive elements as one or two 16-byte transactions.
template <typename T> struct Vec8;

template <> struct Vec8<float> {
    static __device__ __forceinline__ void load(const float *p, float (&v)[8]) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        float4 b = *reinterpret_cast<const float4 *>(p + 4);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
    static __device__ __forceinline__ void store(float *p, const float (&v)[8]) {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4 *>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
};

template <> struct Vec8<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float (&v)[8]) {
        uint4 r = *reinterpret_cast<const uint4 *>(p);
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x;
            v[2 * i + 1] = f.y;
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float (&v)[8]) {
        uint4 r;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&r);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4 *>(p) = r;
    }
};

__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + expf(-v)); }

// Walk-order indexing.  A direction walks steps s = 0 .. len-1; the forward
// stream visits token s, the reverse stream token len-1-s.  Reversal is an
// index reflection: no flipped copy of any tensor is made.
__device__ __forceinline__ int walk_token(int s, int len, bool rev) {
    return rev ? len - 1 - s : s;
}

}  // namespace bimamba
