// conv_staged.cu -- the depthwise conv1d (4 taps) + SiLU of both streams,
// and its backward, as shared-memory-staged tiles for the training path.
//
// Operation: "DiffuMamba" blog post, network-architecture listing
// (d_conv = 4, SiLU after the conv); the reverse stream applies the same conv
// to the reversed sequence ("DiffuMamba" technical summaries, proposed-method
// sections), which in token order is the conv with mirrored taps:
//   pre_f[t] = b + sum_j w_j u[t-3+j],   pre_r[t] = b + sum_j w_j u[t+3-j]
// (zeros outside the sequence).  The backward is the chain rule through
// SiLU and the two convs:
//   du[t] = sum_j w_j dpre_f[t+3-j] + sum_j w_j dpre_r[t-3+j]
//   dw_j  = sum_t dpre_f[t] u[t-3+j] + dpre_r[t] u[t+3-j],  db = sum_t dpre_f[t] + dpre_r[t]
// with dpre = dact * SiLU'(pre).
//
// Both kernels are HBM-bound elementwise passes.  A CTA owns a tile of
// kTileT tokens x kTileC channels: one TMA box per input tensor brings the
// tile with its 3- or 6-token halo into shared memory (rows outside the
// sequence read zeros, so no bounds tests), the compute reads shared
// memory, and the results leave by 8/16-byte stores that a warp issues for
// contiguous 128/256-byte row pieces.  Many small CTAs per SM keep tens of
// kilobytes of loads in flight per SM; a thread walking its channels token
// by token with one 16-byte load at a time keeps only a few.
#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace bimamba {

namespace {

constexpr int kTileT = 64;        // tokens per tile
constexpr int kTileC = 64;        // channels per tile
constexpr int kThreadsSt = 128;   // 16 channel quads x 8 groups of 8 tokens
constexpr long long kStWait = 4000000000LL;   // ~2 s at 1.9 GHz

PFN_cuTensorMapEncodeTiled_v12000 staged_encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// (batch, len, ch) rows, boxes of kTileC channels x `rows` tokens, no swizzle
// (row r of a box at r * kTileC elements in shared memory)
bool make_rows_map(CUtensorMap *m, const void *base, size_t esz, int ch, int len, int batch, int rows)
{
    auto fn = staged_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)ch, (cuuint64_t)len, (cuuint64_t)batch};
    const cuuint64_t strides[2] = {(cuuint64_t)ch * esz, (cuuint64_t)ch * len * esz};
    const cuuint32_t box[3] = {(cuuint32_t)kTileC, (cuuint32_t)rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 4 consecutive channels of a staged row, as floats
template <typename T> __device__ __forceinline__ void lds4(const T *p, float (&v)[4]);
template <> __device__ __forceinline__ void lds4<float>(const float *p, float (&v)[4])
{
    const float4 q = *reinterpret_cast<const float4 *>(p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
}
template <> __device__ __forceinline__ void lds4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[4])
{
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&q.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&q.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

template <typename T> __device__ __forceinline__ void stg4(T *p, const float (&v)[4]);
template <> __device__ __forceinline__ void stg4<float>(float *p, const float (&v)[4])
{
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <> __device__ __forceinline__ void stg4<__nv_bfloat16>(__nv_bfloat16 *p, const float (&v)[4])
{
    *reinterpret_cast<uint2 *>(p) = make_uint2(tc::pack_bf16x2(v[0], v[1]), tc::pack_bf16x2(v[2], v[3]));
}

// SiLU and its derivative, by the activation dtype.  fp32: through the fast
// exponential and divide intrinsics (relative error ~1e-6, inside the fp32
// bound; for x -> -inf, 1 + e^-x overflows to inf and both give (-)0).
// bf16: through the hardware tanh, sigma(x) = 1/2 + tanh(x/2)/2 (relative
// error ~1e-3 in sigma, far inside the bf16 bound), one special-function
// operation instead of two.  With the IEEE expf and division the conv
// passes were bound by these instructions rather than by HBM.
template <typename T> struct Act;
template <> struct Act<float> {
    static __device__ __forceinline__ float silu(float x) { return __fdividef(x, 1.0f + __expf(-x)); }
    static __device__ __forceinline__ float dsilu(float x)
    {
        const float sg = __fdividef(1.0f, 1.0f + __expf(-x));
        return sg * (1.0f + x * (1.0f - sg));
    }
};
template <> struct Act<__nv_bfloat16> {
    static __device__ __forceinline__ float tanh_approx(float x)
    {
        float t;
        asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x));
        return t;
    }
    // x sigma(x) = h + h tanh(h), h = x / 2
    static __device__ __forceinline__ float silu(float x)
    {
        const float h = 0.5f * x;
        return fmaf(h, tanh_approx(h), h);
    }
    static __device__ __forceinline__ float dsilu(float x)
    {
        const float sg = fmaf(0.5f, tanh_approx(0.5f * x), 0.5f);
        return sg * (1.0f + x * (1.0f - sg));
    }
};

// One thread issues the tile's TMA boxes onto one mbarrier; every thread
// waits (bounded).  Returns false on timeout (recorded in the status word).
__device__ __forceinline__ bool wait_tile(uint32_t mb, int *status)
{
    bool ok = tc::mbar_wait_bounded(mb, 0, kStWait);
    if (!ok) record_error(status, kStatusTimeout);
    return __syncthreads_and(ok);
}

}  // namespace

// Both streams' conv + SiLU in token order, from one staged tile of raw rows
// [t0-3, t0+kTileT+3): thread (quad q, group g) produces tokens 8g..8g+7 of
// the tile for channels 4q..4q+3 with a 7-row window.  The fused
// multiply-adds run in the order of conv_silu_kernel's forward and reverse
// instances.
template <typename T>
__global__ void __launch_bounds__(kThreadsSt, 7)
conv_silu_both_staged_kernel(const __grid_constant__ CUtensorMap tm_u, T *__restrict__ out_f,
                             T *__restrict__ out_r, const float *__restrict__ w, const float *__restrict__ bias,
                             int len, int ch, int *status)
{
    constexpr int kRows = kTileT + 6;
    __shared__ alignas(128) T raw[kRows * kTileC];
    __shared__ alignas(8) uint64_t mbar;
    const int tid = threadIdx.x, q = tid & 15, g = tid >> 4;
    const int cb = blockIdx.x * kTileC, t0 = blockIdx.y * kTileT, b = blockIdx.z;
    const uint32_t mb = tc::smem_u32(&mbar);
    if (tid == 0) {
        tc::mbar_init(mb, 1);
        tc::mbar_expect_tx(mb, (uint32_t)sizeof(raw));
        tc::tma_load_3d(tc::smem_u32(raw), &tm_u, cb, t0 - 3, b, mb);
    }
    const int c = cb + 4 * q;
    float wt[4][4], bb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 v = c + k < ch ? *reinterpret_cast<const float4 *>(w + (size_t)(c + k) * 4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        wt[k][0] = v.x; wt[k][1] = v.y; wt[k][2] = v.z; wt[k][3] = v.w;
        bb[k] = (bias && c + k < ch) ? bias[c + k] : 0.0f;
    }
    __syncthreads();   // mbarrier initialised
    if (!wait_tile(mb, status)) return;
    // window x[k] = u[t - 3 + k], k = 0..6; raw row r holds token t0 - 3 + r
    const int i0 = 8 * g;
    float x[7][4];
#pragma unroll
    for (int k = 0; k < 6; ++k) lds4<T>(raw + (i0 + k) * kTileC + 4 * q, x[k]);
    const size_t base = ((size_t)b * len + t0) * ch + c;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        lds4<T>(raw + (i0 + i + 6) * kTileC + 4 * q, x[6]);
        float of[4], orr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float af = bb[k];
            af = fmaf(wt[k][0], x[0][k], af);
            af = fmaf(wt[k][1], x[1][k], af);
            af = fmaf(wt[k][2], x[2][k], af);
            af = fmaf(wt[k][3], x[3][k], af);
            float ar = bb[k];
            ar = fmaf(wt[k][0], x[6][k], ar);
            ar = fmaf(wt[k][1], x[5][k], ar);
            ar = fmaf(wt[k][2], x[4][k], ar);
            ar = fmaf(wt[k][3], x[3][k], ar);
            of[k] = Act<T>::silu(af);
            orr[k] = Act<T>::silu(ar);
        }
        if (t0 + i0 + i < len && c < ch) {
            stg4<T>(out_f + base + (size_t)(i0 + i) * ch, of);
            stg4<T>(out_r + base + (size_t)(i0 + i) * ch, orr);
        }
#pragma unroll
        for (int k = 0; k < 6; ++k)
#pragma unroll
            for (int e = 0; e < 4; ++e) x[k][e] = x[k + 1][e];
    }
}

// The conv backward of both streams from three staged tiles: raw u rows
// [t0-3, t0+kTileT+3), dact_f rows [t0, t0+kTileT+3) and dact_r rows
// [t0-3, t0+kTileT).  Phase 1 turns the dact rows into dpre in place (row r
// of both uses raw rows r..r+3); phase 2 forms du of the tile's tokens and
// the tap / bias gradients, summed over the CTA's token groups in shared
// memory and added once per channel and CTA.
template <typename T>
__global__ void __launch_bounds__(kThreadsSt)
bwd_conv_staged_kernel(const __grid_constant__ CUtensorMap tm_u, const __grid_constant__ CUtensorMap tm_af,
                       const __grid_constant__ CUtensorMap tm_ar, const float *__restrict__ w,
                       const float *__restrict__ bias, float *__restrict__ du, float *__restrict__ dw,
                       float *__restrict__ db, int len, int ch, int *status)
{
    constexpr int kURows = kTileT + 6, kDRows = kTileT + 3;
    extern __shared__ __align__(128) uint8_t smem_st[];
    float *pf = reinterpret_cast<float *>(smem_st);   // dact_f -> dpre_f, row r = token t0 + r
    float *pr = pf + kDRows * kTileC;                 // dact_r -> dpre_r, row r = token t0 - 3 + r
    T *u = reinterpret_cast<T *>(pr + kDRows * kTileC);   // raw, row r = token t0 - 3 + r
    uint64_t *mbar = reinterpret_cast<uint64_t *>(u + kURows * kTileC);
    const int tid = threadIdx.x, q = tid & 15, g = tid >> 4;
    const int cb = blockIdx.x * kTileC, t0 = blockIdx.y * kTileT, b = blockIdx.z;
    const uint32_t mb = tc::smem_u32(mbar);
    if (tid == 0) {
        tc::mbar_init(mb, 1);
        tc::mbar_expect_tx(mb, (uint32_t)(2 * kDRows * kTileC * sizeof(float) + kURows * kTileC * sizeof(T)));
        tc::tma_load_3d(tc::smem_u32(pf), &tm_af, cb, t0, b, mb);
        tc::tma_load_3d(tc::smem_u32(pr), &tm_ar, cb, t0 - 3, b, mb);
        tc::tma_load_3d(tc::smem_u32(u), &tm_u, cb, t0 - 3, b, mb);
    }
    const int c = cb + 4 * q;
    float wc[4][4], bc[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float4 v = c + k < ch ? *reinterpret_cast<const float4 *>(w + (size_t)(c + k) * 4)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        wc[k][0] = v.x; wc[k][1] = v.y; wc[k][2] = v.z; wc[k][3] = v.w;
        bc[k] = (bias && c + k < ch) ? bias[c + k] : 0.0f;
    }
    __syncthreads();   // mbarrier initialised
    if (!wait_tile(mb, status)) return;
    // phase 1: rows r = g, g + 8, ...: pre_f(t0 + r) = b + sum_j w_j u[r + j],
    // pre_r(t0 - 3 + r) = b + sum_j w_j u[r + 3 - j] (rows outside the
    // sequence hold dact = 0, so their dpre is 0)
    for (int r = g; r < kDRows; r += 8) {
        float u0[4], u1[4], u2[4], u3[4], a[4], e[4];
        lds4<T>(u + r * kTileC + 4 * q, u0);
        lds4<T>(u + (r + 1) * kTileC + 4 * q, u1);
        lds4<T>(u + (r + 2) * kTileC + 4 * q, u2);
        lds4<T>(u + (r + 3) * kTileC + 4 * q, u3);
        lds4<float>(pf + r * kTileC + 4 * q, a);
        lds4<float>(pr + r * kTileC + 4 * q, e);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float pre_f = bc[k] + wc[k][0] * u0[k] + wc[k][1] * u1[k] + wc[k][2] * u2[k] + wc[k][3] * u3[k];
            const float pre_r = bc[k] + wc[k][0] * u3[k] + wc[k][1] * u2[k] + wc[k][2] * u1[k] + wc[k][3] * u0[k];
            a[k] *= Act<T>::dsilu(pre_f);
            e[k] *= Act<T>::dsilu(pre_r);
        }
        *reinterpret_cast<float4 *>(pf + r * kTileC + 4 * q) = make_float4(a[0], a[1], a[2], a[3]);
        *reinterpret_cast<float4 *>(pr + r * kTileC + 4 * q) = make_float4(e[0], e[1], e[2], e[3]);
    }
    __syncthreads();
    // phase 2: tokens i = 8g .. 8g+7 of the tile:
    //   du = w0 pf[i+3] + w1 pf[i+2] + w2 pf[i+1] + w3 pf[i] + w0 pr[i] + w1 pr[i+1] + w2 pr[i+2] + w3 pr[i+3]
    //   dw_j += pf[i] u[i+j] + pr[i+3] u[i+6-j] (j < 3), dw_3 += (pf[i] + pr[i+3]) u[i+3]
    float g0[4] = {0, 0, 0, 0}, g1[4] = {0, 0, 0, 0}, g2[4] = {0, 0, 0, 0}, g3[4] = {0, 0, 0, 0},
          gbs[4] = {0, 0, 0, 0};
    const int i0 = 8 * g;
    const size_t base = ((size_t)b * len + t0) * ch + c;
#pragma unroll 2
    for (int i = i0; i < i0 + 8; ++i) {
        float f0[4], f1[4], f2[4], f3[4], r0[4], r1[4], r2[4], r3[4];
        lds4<float>(pf + i * kTileC + 4 * q, f0);
        lds4<float>(pf + (i + 1) * kTileC + 4 * q, f1);
        lds4<float>(pf + (i + 2) * kTileC + 4 * q, f2);
        lds4<float>(pf + (i + 3) * kTileC + 4 * q, f3);
        lds4<float>(pr + i * kTileC + 4 * q, r0);
        lds4<float>(pr + (i + 1) * kTileC + 4 * q, r1);
        lds4<float>(pr + (i + 2) * kTileC + 4 * q, r2);
        lds4<float>(pr + (i + 3) * kTileC + 4 * q, r3);
        float gd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            gd[k] = wc[k][0] * f3[k] + wc[k][1] * f2[k] + wc[k][2] * f1[k] + wc[k][3] * f0[k] +
                    wc[k][0] * r0[k] + wc[k][1] * r1[k] + wc[k][2] * r2[k] + wc[k][3] * r3[k];
        if (t0 + i < len && c < ch) stg4<float>(du + base + (size_t)i * ch, gd);
        float v0[4], v1[4], v2[4], v3[4], v4[4], v5[4], v6[4];
        lds4<T>(u + i * kTileC + 4 * q, v0);
        lds4<T>(u + (i + 1) * kTileC + 4 * q, v1);
        lds4<T>(u + (i + 2) * kTileC + 4 * q, v2);
        lds4<T>(u + (i + 3) * kTileC + 4 * q, v3);
        lds4<T>(u + (i + 4) * kTileC + 4 * q, v4);
        lds4<T>(u + (i + 5) * kTileC + 4 * q, v5);
        lds4<T>(u + (i + 6) * kTileC + 4 * q, v6);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float dpf = f0[k], dpr = r3[k];
            g0[k] += dpf * v0[k] + dpr * v6[k];
            g1[k] += dpf * v1[k] + dpr * v5[k];
            g2[k] += dpf * v2[k] + dpr * v4[k];
            g3[k] += (dpf + dpr) * v3[k];
            gbs[k] += dpf + dpr;
        }
    }
    // the tap and bias gradients: sum the 8 token groups of each channel in
    // shared memory (over the dpre_f rows, which are no longer read), then
    // one atomic add per channel, tap and CTA
    __syncthreads();
    float *red = pf;   // [8 groups][5][kTileC]
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        red[(g * 5 + 0) * kTileC + 4 * q + k] = g0[k];
        red[(g * 5 + 1) * kTileC + 4 * q + k] = g1[k];
        red[(g * 5 + 2) * kTileC + 4 * q + k] = g2[k];
        red[(g * 5 + 3) * kTileC + 4 * q + k] = g3[k];
        red[(g * 5 + 4) * kTileC + 4 * q + k] = gbs[k];
    }
    __syncthreads();
    for (int e = tid; e < 5 * kTileC; e += kThreadsSt) {
        const int v = e / kTileC, cc = e % kTileC;
        if (cb + cc >= ch || (v == 4 && !db)) continue;
        float s = 0.0f;
#pragma unroll
        for (int gg = 0; gg < 8; ++gg) s += red[(gg * 5 + v) * kTileC + cc];
        if (v < 4)
            atomicAdd(dw + (size_t)(cb + cc) * 4 + v, s);
        else
            atomicAdd(db + cb + cc, s);
    }
}

namespace {
constexpr size_t bwd_staged_smem(size_t esz)
{
    return 2 * (kTileT + 3) * kTileC * sizeof(float) + (kTileT + 6) * kTileC * esz + 16;
}
}  // namespace

template <typename T>
cudaError_t launch_conv_silu_both_staged(const void *u, void *out_f, void *out_r, const float *w,
                                         const float *bias, int batch, int len, int ch, cudaStream_t stream)
{
    CUtensorMap tm;
    if (!make_rows_map(&tm, u, sizeof(T), ch, len, batch, kTileT + 6)) return cudaErrorInvalidValue;
    const dim3 grid((ch + kTileC - 1) / kTileC, (len + kTileT - 1) / kTileT, batch);
    conv_silu_both_staged_kernel<T><<<grid, kThreadsSt, 0, stream>>>(
        tm, static_cast<T *>(out_f), static_cast<T *>(out_r), w, bias, len, ch, device_status_word());
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template <typename T>
cudaError_t launch_bwd_conv_staged(const void *u, const float *w, const float *bias, const float *dact_f,
                                   const float *dact_r, float *du, float *dw, float *db, int batch, int len,
                                   int ch, cudaStream_t stream)
{
    CUtensorMap tu, tf, tr;
    if (!make_rows_map(&tu, u, sizeof(T), ch, len, batch, kTileT + 6) ||
        !make_rows_map(&tf, dact_f, 4, ch, len, batch, kTileT + 3) ||
        !make_rows_map(&tr, dact_r, 4, ch, len, batch, kTileT + 3))
        return cudaErrorInvalidValue;
    const size_t smem = bwd_staged_smem(sizeof(T));
    cudaError_t e = cudaFuncSetAttribute(bwd_conv_staged_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((ch + kTileC - 1) / kTileC, (len + kTileT - 1) / kTileT, batch);
    bwd_conv_staged_kernel<T><<<grid, kThreadsSt, smem, stream>>>(tu, tf, tr, w, bias, du, dw, db, len, ch,
                                                                   device_status_word());
    e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

template cudaError_t launch_conv_silu_both_staged<float>(const void *, void *, void *, const float *,
                                                         const float *, int, int, int, cudaStream_t);
template cudaError_t launch_conv_silu_both_staged<__nv_bfloat16>(const void *, void *, void *, const float *,
                                                                 const float *, int, int, int, cudaStream_t);
template cudaError_t launch_bwd_conv_staged<float>(const void *, const float *, const float *, const float *,
                                                   const float *, float *, float *, float *, int, int, int,
                                                   cudaStream_t);
template cudaError_t launch_bwd_conv_staged<__nv_bfloat16>(const void *, const float *, const float *,
                                                           const float *, const float *, float *, float *,
                                                           float *, int, int, int, cudaStream_t);

}  // namespace bimamba
