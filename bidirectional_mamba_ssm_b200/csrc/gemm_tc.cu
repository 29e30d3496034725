// gemm_tc.cu -- the projections on either side of the mixer, on the sm_100a
// tensor cores: a persistent tcgen05 GEMM  C = A . W^T  (bf16 operands, fp32
// accumulators in tensor memory) whose epilogue writes the mixer's own
// input layouts.
//
// Sources: "DiffuMamba" blog post, network-architecture listing (d_model =
// 2048, expand = 2: each Mamba mixer maps d_model to its inner width and
// back; the bidirectional block concatenates its two streams and maps 2d
// back to d with a Linear); the Mamba-2 block's input projection produces
// the conv input xBC and the step sizes dt = softplus(raw + dt_bias).
//   in-projection : [xbc | dt_raw] = u . W_in^T, dt = softplus(dt_raw + b)
//                   written straight into the (tokens, ch) and (tokens, H)
//                   tensors bimamba_ssd_fwd_rev reads
//   out-projection: out = y . W_out^T, reading the mixer's y (summed, or the
//                   concatenation [forward | reverse] of untied directions)
//
// Kernel: one CTA per SM walks output tiles of 128 x 256 (M x N) in a
// persistent loop.  Warp 0 streams 64-deep K slices of A and W by TMA into a
// 4-stage ring (48 KB per stage, 128-byte swizzle); warp 1 issues the
// tcgen05 MMAs (M = 128, N = 256, K = 16) into one of two 256-column
// accumulators; warps 2..5 drain the other accumulator (tcgen05.ld, the
// epilogue, global stores) while the next tile accumulates.  Every wait is
// bounded; a wait that gives up records BIMAMBA_ERR_TIMEOUT and ends the CTA.
#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

namespace bimamba {

namespace {

constexpr int kGM = 128, kGN = 256, kGK = 64;
constexpr int kGStages = 4;
constexpr uint32_t kGStageA = kGM * kGK * 2;   // 16 KB
constexpr uint32_t kGStageB = kGN * kGK * 2;   // 32 KB
constexpr uint32_t kGStage = kGStageA + kGStageB;
constexpr uint32_t kGOffBar = kGStages * kGStage;   // 192 KB of operand ring
constexpr uint32_t kGOffTmem = kGOffBar + 12 * 8;
constexpr uint32_t kGSmem = kGOffTmem + 16 + 1024;
constexpr int kGThreads = 192;
constexpr long long kGWait = 4000000000LL;   // ~2 s at 1.9 GHz

struct GemmParams {
    int M, N, K;
    // columns [0, n_split) -> out0 (row stride n_split), bf16;
    // columns [n_split, N) -> out1 (row stride N - n_split), bf16 of
    // softplus(acc + bias1[c - n_split]) (bias1 may be null)
    int n_split;
    __nv_bfloat16 *out0, *out1;
    const float *bias1;
    int *status;
};

__device__ __forceinline__ float softplus_f(float x)
{
    return x > 20.0f ? x : log1pf(expf(x));
}

}  // namespace

__global__ void __launch_bounds__(kGThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
               const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int mblocks = (p.M + kGM - 1) / kGM, nblocks = (p.N + kGN - 1) / kGN;
    const int tiles = mblocks * nblocks;
    const int ksteps = (p.K + kGK - 1) / kGK;
    const uint32_t bar = sbase + kGOffBar;
    auto full = [&](int s) { return bar + 8 * s; };                   // stage s landed
    auto empty = [&](int s) { return bar + 8 * (kGStages + s); };     // stage s consumed
    auto accf = [&](int j) { return bar + 8 * (2 * kGStages + j); };  // accumulator j done
    auto acce = [&](int j) { return bar + 8 * (2 * kGStages + 2 + j); };   // accumulator j drained

    if (tid == 0) {
        tc::prefetch_tmap(&tm_a);
        tc::prefetch_tmap(&tm_b);
        for (int s = 0; s < kGStages; ++s) {
            tc::mbar_init(full(s), 1);
            tc::mbar_init(empty(s), 1);
        }
        for (int j = 0; j < 2; ++j) {
            tc::mbar_init(accf(j), 1);
            tc::mbar_init(acce(j), 4);   // one arrival per epilogue warp
        }
    }
    if (warp == 1) tc::tmem_alloc(sbase + kGOffTmem, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kGOffTmem);

    if (warp == 0) {
        // ---- TMA producer (lane 0)
        if (lane == 0) {
            bool ok = true;
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
                const int mb = tile / nblocks, nb = tile % nblocks;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = (it / kGStages) & 1;
                    if (!(ok = tc::mbar_wait_bounded(empty(s), ph ^ 1, kGWait))) break;
                    tc::mbar_expect_tx(full(s), kGStage);
                    const uint32_t dst = sbase + s * kGStage;
                    tc::tma_load_2d(dst, &tm_a, ks * kGK, mb * kGM, full(s));
                    tc::tma_load_2d(dst + kGStageA, &tm_b, ks * kGK, nb * kGN, full(s));
                }
            }
            if (!ok) record_error(p.status, kStatusTimeout);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---- MMA issuer (lane 0)
        if (lane == 0) {
            constexpr uint32_t idesc = tc::idesc_bf16(kGM, kGN, 0, 0);
            bool ok = true;
            uint32_t it = 0, tcount = 0;
            for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tcount) {
                const int j = tcount & 1;
                const uint32_t use = tcount >> 1;
                if (!(ok = tc::mbar_wait_bounded(acce(j), (use & 1) ^ 1, kGWait))) break;
                tc::fence_after_sync();
                const uint32_t acc = tmem + kGN * j;
                for (int ks = 0; ks < ksteps; ++ks, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = (it / kGStages) & 1;
                    if (!(ok = tc::mbar_wait_bounded(full(s), ph, kGWait))) break;
                    tc::fence_after_sync();
                    const uint64_t da = tc::smem_desc(sbase + s * kGStage, 16, 1024);
                    const uint64_t db = tc::smem_desc(sbase + s * kGStage + kGStageA, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < kGK / 16; ++kk)
                        tc::mma_bf16(acc, tc::desc_add(da, 32 * kk), tc::desc_add(db, 32 * kk), idesc,
                                     (ks | kk) != 0);
                    tc::mma_commit(empty(s));   // the stage is free once these MMAs complete
                }
                if (ok) tc::mma_commit(accf(j));
            }
            if (!ok) record_error(p.status, kStatusTimeout);
        }
        __syncwarp();
    } else {
        // ---- epilogue (warps 2..5; warp w reads TMEM lanes 32 (w % 4) ..)
        const int q = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * q) << 16;
        uint32_t tcount = 0;
        bool ok = true;
        const int n1 = p.N - p.n_split;
        for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++tcount) {
            const int mb = tile / nblocks, nb = tile % nblocks;
            const int j = tcount & 1;
            const uint32_t use = tcount >> 1;
            if (lane == 0) ok = tc::mbar_wait_bounded(accf(j), use & 1, kGWait);
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc::fence_after_sync();
            const int row = mb * kGM + 32 * q + lane;
            for (int c32 = 0; c32 < kGN / 32; ++c32) {
                const int col0 = nb * kGN + 32 * c32;
                if (col0 >= p.N) break;   // warp-uniform
                float v[32];
                tc::tmem_ld32(tmem + lane_base + kGN * j + 32 * c32, v);
                if (row >= p.M) continue;
                if (col0 + 32 <= p.n_split && (p.n_split & 7) == 0) {
                    // the whole chunk in out0, 16-byte stores
                    uint4 *dst = reinterpret_cast<uint4 *>(p.out0 + (size_t)row * p.n_split + col0);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 w;
                        w.x = tc::pack_bf16x2(v[8 * i], v[8 * i + 1]);
                        w.y = tc::pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
                        w.z = tc::pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
                        w.w = tc::pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
                        dst[i] = w;
                    }
                } else {
                    for (int i = 0; i < 32; ++i) {
                        const int c = col0 + i;
                        if (c >= p.N) break;
                        if (c < p.n_split) {
                            p.out0[(size_t)row * p.n_split + c] = __float2bfloat16_rn(v[i]);
                        } else {
                            const int cc = c - p.n_split;
                            const float x = v[i] + (p.bias1 ? p.bias1[cc] : 0.0f);
                            p.out1[(size_t)row * n1 + cc] = __float2bfloat16_rn(softplus_f(x));
                        }
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(acce(j));   // the accumulator may be reused
        }
        if (!ok && lane == 0) record_error(p.status, kStatusTimeout);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 gemm_encode_fn()
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

// 2-D bf16 row-major (rows, K) operand, box (64, box_rows), 128-byte swizzle
bool make_operand_map(CUtensorMap *m, const void *base, uint64_t K, uint64_t rows, uint32_t box_rows)
{
    auto fn = gemm_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kGK, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_gemm_tc(const GemmProblem &g, cudaStream_t stream)
{
    CUtensorMap ta, tb;
    if (!make_operand_map(&ta, g.a, (uint64_t)g.K, (uint64_t)g.M, kGM) ||
        !make_operand_map(&tb, g.w, (uint64_t)g.K, (uint64_t)g.N, kGN))
        return cudaErrorInvalidValue;
    GemmParams p;
    p.M = g.M;
    p.N = g.N;
    p.K = g.K;
    p.n_split = g.n_split;
    p.out0 = static_cast<__nv_bfloat16 *>(g.out0);
    p.out1 = static_cast<__nv_bfloat16 *>(g.out1);
    p.bias1 = g.bias1;
    p.status = g.status;
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kGSmem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long tiles = (long long)((g.M + kGM - 1) / kGM) * ((g.N + kGN - 1) / kGN);
    const int grid = (int)std::min<long long>(tiles, sms);
    const TimingEvents ev = timing_events();
    if (ev.start && (e = cudaEventRecord(ev.start, stream)) != cudaSuccess) return e;
    gemm_tc_kernel<<<grid, kGThreads, kGSmem, stream>>>(ta, tb, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    if (ev.stop) e = cudaEventRecord(ev.stop, stream);
    return e;
}

}  // namespace bimamba
