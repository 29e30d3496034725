// conv_silu.cu -- stand-alone depthwise conv1d (4 taps) + SiLU, causal or
// mirrored (reverse stream), for the bidirectional Mamba-2 mixer.
//
// Operation: "DiffuMamba" blog post, network-architecture listing
// (d_conv = 4); the reverse stream is the same conv on the reversed sequence
// ("DiffuMamba" technical summaries, proposed-method sections), done here by
// index reflection.
//
// Layout: u/out (batch, len, ch) token-major, channel-contiguous.  One thread
// owns 8 consecutive channels (one 16-byte load for bf16, two for fp32) and a
// tile of kTile walk steps, keeping the 3-token window in registers, so each
// input element is read once per tile plus a 3-token halo.  HBM-bound:
// 2 * ch * sizeof(T) bytes per token.
#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

constexpr int kConvTile = 64;

template <typename T>
__global__ void __launch_bounds__(128)
conv_silu_kernel(const T *__restrict__ u, T *__restrict__ out, const float *__restrict__ w,
                 const float *__restrict__ bias, const T *__restrict__ tail, int len, int ch,
                 int rev, int silu)
{
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (c0 >= ch) return;
    const int b = blockIdx.z;
    const int s0 = blockIdx.y * kConvTile;
    const int s1 = min(s0 + kConvTile, len);
    const T *ub = u + (size_t)b * len * ch + c0;
    T *ob = out + (size_t)b * len * ch + c0;

    float wt[8][4], bb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float4 q = *reinterpret_cast<const float4 *>(w + (size_t)(c0 + i) * 4);
        wt[i][0] = q.x; wt[i][1] = q.y; wt[i][2] = q.z; wt[i][3] = q.w;
        bb[i] = bias ? bias[c0 + i] : 0.0f;
    }

    // raw value at walk step s (s may be -3..-1: the halo before the start)
    auto load_raw = [&](int s, float (&v)[8]) {
        if (s >= 0) {
            Vec8<T>::load(ub + (size_t)walk_token(s, len, rev) * ch, v);
        } else if (!rev && tail) {
            Vec8<T>::load(tail + ((size_t)b * 4 + (4 + s)) * ch + c0, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
    };

    float r0[8], r1[8], r2[8];
    load_raw(s0 - 3, r0);
    load_raw(s0 - 2, r1);
    load_raw(s0 - 1, r2);
    for (int s = s0; s < s1; ++s) {
        float r3[8], o[8];
        load_raw(s, r3);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float acc = bb[i];
            acc = fmaf(wt[i][0], r0[i], acc);
            acc = fmaf(wt[i][1], r1[i], acc);
            acc = fmaf(wt[i][2], r2[i], acc);
            acc = fmaf(wt[i][3], r3[i], acc);
            o[i] = silu ? silu_f(acc) : acc;
            r0[i] = r1[i]; r1[i] = r2[i]; r2[i] = r3[i];
        }
        Vec8<T>::store(ob + (size_t)walk_token(s, len, rev) * ch, o);
    }
}

template <typename T>
cudaError_t launch_conv_silu(const void *u, void *out, const float *w, const float *bias,
                             const void *tail, int batch, int len, int ch, int rev, int silu,
                             cudaStream_t stream)
{
    dim3 block(128);
    dim3 grid((ch / 8 + 127) / 128, (len + kConvTile - 1) / kConvTile, batch);
    conv_silu_kernel<T><<<grid, block, 0, stream>>>(
        static_cast<const T *>(u), static_cast<T *>(out), w, bias,
        static_cast<const T *>(tail), len, ch, rev, silu);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

template cudaError_t launch_conv_silu<float>(const void *, void *, const float *, const float *,
                                             const void *, int, int, int, int, int, cudaStream_t);
template cudaError_t launch_conv_silu<__nv_bfloat16>(const void *, void *, const float *,
                                                     const float *, const void *, int, int, int,
                                                     int, int, cudaStream_t);

}  // namespace bimamba
