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

// Both streams' conv + SiLU of one raw input (tied taps), in token order:
// out_f[t] = SiLU(b + sum_j w_j u[t-3+j]), out_r[t] = SiLU(b + sum_j w_j u[t+3-j])
// (zeros outside the sequence; the same arithmetic, in the same order, as
// conv_silu_kernel's forward and reverse instances).  Each raw row is read
// once for both: one thread owns 8 channels and a tile of kConvTile tokens
// with a 7-row window.
template <typename T>
__global__ void __launch_bounds__(128)
conv_silu_both_kernel(const T *__restrict__ u, T *__restrict__ out_f, T *__restrict__ out_r,
                      const float *__restrict__ w, const float *__restrict__ bias, int len, int ch)
{
    const int c0 = (blockIdx.x * blockDim.x + threadIdx.x) * 8;
    if (c0 >= ch) return;
    const int b = blockIdx.z;
    const int t0 = blockIdx.y * kConvTile;
    const int t1 = min(t0 + kConvTile, len);
    const T *ub = u + (size_t)b * len * ch + c0;
    T *of = out_f + (size_t)b * len * ch + c0;
    T *orr = out_r + (size_t)b * len * ch + c0;
    float wt[8][4], bb[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float4 q = *reinterpret_cast<const float4 *>(w + (size_t)(c0 + i) * 4);
        wt[i][0] = q.x; wt[i][1] = q.y; wt[i][2] = q.z; wt[i][3] = q.w;
        bb[i] = bias ? bias[c0 + i] : 0.0f;
    }
    auto load_raw = [&](int t, float (&v)[8]) {
        if (t >= 0 && t < len) {
            Vec8<T>::load(ub + (size_t)t * ch, v);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) v[i] = 0.0f;
        }
    };
    // window: x0..x6 = u[t-3 .. t+3]
    float x0[8], x1[8], x2[8], x3[8], x4[8], x5[8];
    load_raw(t0 - 3, x0);
    load_raw(t0 - 2, x1);
    load_raw(t0 - 1, x2);
    load_raw(t0, x3);
    load_raw(t0 + 1, x4);
    load_raw(t0 + 2, x5);
    for (int t = t0; t < t1; ++t) {
        float x6[8], of8[8], or8[8];
        load_raw(t + 3, x6);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float af = bb[i];
            af = fmaf(wt[i][0], x0[i], af);
            af = fmaf(wt[i][1], x1[i], af);
            af = fmaf(wt[i][2], x2[i], af);
            af = fmaf(wt[i][3], x3[i], af);
            float ar = bb[i];
            ar = fmaf(wt[i][0], x6[i], ar);
            ar = fmaf(wt[i][1], x5[i], ar);
            ar = fmaf(wt[i][2], x4[i], ar);
            ar = fmaf(wt[i][3], x3[i], ar);
            of8[i] = silu_f(af);
            or8[i] = silu_f(ar);
            x0[i] = x1[i]; x1[i] = x2[i]; x2[i] = x3[i]; x3[i] = x4[i]; x4[i] = x5[i]; x5[i] = x6[i];
        }
        Vec8<T>::store(of + (size_t)t * ch, of8);
        Vec8<T>::store(orr + (size_t)t * ch, or8);
    }
}

template <typename T>
cudaError_t launch_conv_silu_both(const void *u, void *out_f, void *out_r, const float *w, const float *bias,
                                  int batch, int len, int ch, cudaStream_t stream)
{
    dim3 block(128);
    dim3 grid((ch / 8 + 127) / 128, (len + kConvTile - 1) / kConvTile, batch);
    conv_silu_both_kernel<T><<<grid, block, 0, stream>>>(static_cast<const T *>(u), static_cast<T *>(out_f),
                                                          static_cast<T *>(out_r), w, bias, len, ch);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

template cudaError_t launch_conv_silu_both<float>(const void *, void *, void *, const float *, const float *, int,
                                                  int, int, cudaStream_t);
template cudaError_t launch_conv_silu_both<__nv_bfloat16>(const void *, void *, void *, const float *,
                                                          const float *, int, int, int, cudaStream_t);

template cudaError_t launch_conv_silu<float>(const void *, void *, const float *, const float *,
                                             const void *, int, int, int, int, int, cudaStream_t);
template cudaError_t launch_conv_silu<__nv_bfloat16>(const void *, void *, const float *,
                                                     const float *, const void *, int, int, int,
                                                     int, int, cudaStream_t);

}  // namespace bimamba
