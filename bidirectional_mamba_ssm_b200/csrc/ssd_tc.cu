// ssd_tc.cu -- chunked bidirectional SSD scan on the sm_100a tensor cores
// (tcgen05 MMAs with fp32 accumulators in tensor memory), conv+SiLU fused
// into the operand staging, reverse direction by index reflection, and the
// forward+reverse sum fused into the epilogue.
//
// Operation (per head h, A_h < 0; "DiffuMamba: High-Throughput Diffusion LMs
// with Mamba Backbone", technical summaries, proposed-method sections: a
// bidirectional Mamba-2 mixer, forward and reverse streams added; d_conv = 4
// from the "DiffuMamba" blog's network-architecture listing):
//     h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T,   y_t = h_t C_t + D_h x_t
//
// Chunked form used here (chunks of Q = 128 walk steps; c_j = inclusive
// prefix sum of dt*A inside the chunk; S_in = state entering the chunk):
//     G      = C B^T                                  (Q x Q,  K = N)
//     M[t,s] = G[t,s] exp(c_t - c_s) dt_s  for s <= t, else 0
//     Y      = M X + diag(exp(c)) C S_in^T + D X     (Q x P)
//     S_out  = exp(c_last) S_in + sum_s exp(c_last - c_s) dt_s x_s B_s^T
// The reverse stream is the same computation in walk order: chunk slots map
// to tokens through t = len-1-s; no flipped copy of any tensor is made.
//
// Mapping: one CTA (256 threads) owns (batch b, head h, direction) and walks
// the chunks of its sequence; the fp32 state lives in registers (thread
// (n, half) holds S[32*half .. 32*half+31][n]); per chunk four MMAs run with
// M = 128 (all products are 128 x 128 x {128, 64}):
//     G        = C  . B^T      A = C  [t][n] K-major,  B = B  [s][n] K-major
//     Y_diag   = M  . X        A = M  [t][s] K-major,  B = X  [s][p] MN-major
//     Y_off    = C  . S_in^T   A = C  [t][n] K-major,  B = S^T[n][p] MN-major
//     dS^T     = B^T. (wX)     A = B  [s][n] MN-major, B = wX [s][p] MN-major
// TMEM: G in columns 0..127 (reused by Y_diag 0..63 and Y_off 64..127 once M
// is built), dS^T in 128..191.
// Descriptors: K-major operands use stride 1024 B between 8-row groups; an
// MN-major operand uses leading offset = distance between its 64-element
// blocks along M/N (16 KB for the 128-wide B tile; the 64-wide tiles have a
// single block, where the field is unused and set equal to the 1024 B stride)
// and stride offset = 1024 B between groups of 8 rows along K.
//
// Forward+reverse sum: the two CTAs of a (b, h) pair meet per token chunk
// through a two-counter handshake in the caller's workspace: the first to
// finish a chunk writes its output (bf16), the second adds its own to it.
// The second one's wait is bounded; the first never waits.
#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

namespace bimamba {

namespace {

constexpr int kQ = 128;  // chunk length
constexpr int kP = 64;   // headdim of this kernel
constexpr int kN = 128;  // d_state of this kernel
constexpr int kThreads = 256;
constexpr int kLocalCh = kP + 2 * kN;  // channels one CTA reads: x of its head, B, C
constexpr uint32_t kTmemCols = 256;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;        // C      [t][n]   2 x 16 KB blocks
constexpr uint32_t kOffB = 32768;    // B      [s][n]   2 x 16 KB
constexpr uint32_t kOffM = 65536;    // M      [t][s]   2 x 16 KB
constexpr uint32_t kOffX = 98304;    // X      [s][p]   16 KB
constexpr uint32_t kOffXw = 114688;  // wX     [s][p]   16 KB
constexpr uint32_t kOffS = 131072;   // S^T    [n][p]   16 KB (bf16 copy)
constexpr uint32_t kOffCum = 147456;            // f32[128] prefix sums of dt*A
constexpr uint32_t kOffDt = kOffCum + 512;      // f32[128] dt
constexpr uint32_t kOffW = kOffDt + 512;        // f32[128] exp(c_last - c_s) dt_s
constexpr uint32_t kOffConvW = kOffW + 512;     // float4[320] conv taps
constexpr uint32_t kOffConvB = kOffConvW + 16 * kLocalCh;  // f32[320]
constexpr uint32_t kOffWsum = kOffConvB + 4 * kLocalCh;     // f32[8] warp sums
constexpr uint32_t kOffMbar = kOffWsum + 64;    // u64 mbarrier
constexpr uint32_t kOffTmem = kOffMbar + 8;     // u32 TMEM base
constexpr uint32_t kOffFlag = kOffTmem + 4;     // i32 handshake result
constexpr uint32_t kSmemUsed = kOffFlag + 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;  // + alignment slack

constexpr uint32_t kColG = 0;
constexpr uint32_t kColYd = 0;
constexpr uint32_t kColYo = 64;
constexpr uint32_t kColDS = 128;

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz

struct TcParams {
    const __nv_bfloat16 *xbc;
    const __nv_bfloat16 *dt;
    const float *A;
    const float *D;
    const float *conv_w;
    const float *conv_b;
    const __nv_bfloat16 *tail;
    const float *init;
    float *fin;
    __nv_bfloat16 *y;
    int *flags;   // [batch][H][nchunks][2]: arrivals, partial-ready
    int *status;
    int len, H, ch, nchunks;
};

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void unpack8(uint4 r, float (&v)[8])
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float *v)
{
    uint4 r;
    r.x = tc::pack_bf16x2(v[0], v[1]);
    r.y = tc::pack_bf16x2(v[2], v[3]);
    r.z = tc::pack_bf16x2(v[4], v[5]);
    r.w = tc::pack_bf16x2(v[6], v[7]);
    return r;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) ssd_tc_kernel(const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x >> 1;
    const bool rev = (blockIdx.x & 1) != 0;
    const int b = blockIdx.y;
    const int H = p.H, L = p.len, ch = p.ch;

    float *cum = reinterpret_cast<float *>(sm + kOffCum);
    float *dts = reinterpret_cast<float *>(sm + kOffDt);
    float *wgt = reinterpret_cast<float *>(sm + kOffW);
    float4 *convw = reinterpret_cast<float4 *>(sm + kOffConvW);
    float *convb = reinterpret_cast<float *>(sm + kOffConvB);
    float *wsum = reinterpret_cast<float *>(sm + kOffWsum);
    int *flag_slot = reinterpret_cast<int *>(sm + kOffFlag);
    const uint32_t mbar = sbase + kOffMbar;

    // ---- setup: conv taps of this CTA's channels, TMEM, mbarrier
    const bool has_conv = p.conv_w != nullptr;
    for (int lc = tid; lc < kLocalCh; lc += kThreads) {
        const int c = lc < kP ? h * kP + lc : H * kP + (lc - kP);
        if (has_conv) {
            convw[lc] = *reinterpret_cast<const float4 *>(p.conv_w + (size_t)c * 4);
            convb[lc] = p.conv_b ? p.conv_b[c] : 0.0f;
        }
    }
    if (warp == 0) tc::tmem_alloc(sbase + kOffTmem, kTmemCols);
    if (tid == 0) tc::mbar_init(mbar, 1);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kOffTmem);

    const int row = tid & 127;   // TMEM lane = tile row this thread serves
    const int half = tid >> 7;   // which 32-column half of a 64-wide result
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float Ah = p.A[h], Dh = p.D[h];
    const size_t sidx = ((size_t)b * H + h) * kP * kN;

    // ---- state: S^T[n = row][p = 32*half + k], fp32 in registers
    float S[32];
#pragma unroll
    for (int k = 0; k < 32; ++k)
        S[k] = (!rev && p.init) ? p.init[sidx + (size_t)(32 * half + k) * kN + row] : 0.0f;
    auto store_state_bf16 = [&]() {
        uint8_t *Sb = sm + kOffS;
#pragma unroll
        for (int pc = 0; pc < 4; ++pc)
            *reinterpret_cast<uint4 *>(Sb + tc::sw128(row, 4 * half + pc)) = pack8(S + 8 * pc);
    };
    store_state_bf16();

    const __nv_bfloat16 *xb = p.xbc + (size_t)b * L * ch;
    const __nv_bfloat16 *tailb = p.tail ? p.tail + (size_t)b * 4 * ch : nullptr;
    uint32_t phase = 0;
    bool ok = true;

    for (int k = 0; k < p.nchunks; ++k) {
        const int c = rev ? p.nchunks - 1 - k : k;  // token chunk
        const int t0 = c * kQ;
        const int cnt = min(kQ, L - t0);
        const int s0 = rev ? L - t0 - cnt : t0;     // walk step of slot 0

        // ---- A: dt, inclusive prefix sums of dt*A, state weights
        if (tid < kQ) {
            float d = 0.0f;
            if (tid < cnt) {
                const int s = s0 + tid;
                const int tok = rev ? L - 1 - s : s;
                d = __bfloat162float(p.dt[((size_t)b * L + tok) * H + h]);
            }
            float a = d * Ah;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, a, o);
                if (lane >= o) a += v;
            }
            if (lane == 31) wsum[warp] = a;
            dts[tid] = d;
            cum[tid] = a;
        }
        __syncthreads();
        if (tid < kQ) {
            float off = 0.0f;
            for (int w = 0; w < (tid >> 5); ++w) off += wsum[w];
            cum[tid] += off;
        }
        __syncthreads();
        const float cum_last = cum[kQ - 1];
        if (tid < kQ) wgt[tid] = __expf(cum_last - cum[tid]) * dts[tid];
        __syncthreads();

        // ---- B: conv+SiLU of x (this head), B, C into the swizzled tiles
        for (int it = tid; it < (kLocalCh / 8) * (kQ / 8); it += kThreads) {
            const int g = it % (kLocalCh / 8), r = it / (kLocalCh / 8);
            const int j0 = r * 8;
            const int lc0 = 8 * g;
            const int cg = lc0 < kP ? h * kP + lc0 : H * kP + (lc0 - kP);
            float o[8][8];
            if (j0 >= cnt) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int q = 0; q < 8; ++q) o[i][q] = 0.0f;
            } else {
                auto raw = [&](int j, float (&v)[8]) {
                    const int s = s0 + j;
                    if (s >= 0) {
                        const int tok = rev ? L - 1 - s : s;
                        unpack8(*reinterpret_cast<const uint4 *>(xb + (size_t)tok * ch + cg), v);
                    } else if (!rev && tailb) {
                        unpack8(*reinterpret_cast<const uint4 *>(tailb + (size_t)(4 + s) * ch + cg), v);
                    } else {
#pragma unroll
                        for (int q = 0; q < 8; ++q) v[q] = 0.0f;
                    }
                };
                if (has_conv) {
                    float w0[8], w1[8], w2[8], w3[8], bb[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 t4 = convw[lc0 + q];
                        w0[q] = t4.x; w1[q] = t4.y; w2[q] = t4.z; w3[q] = t4.w;
                        bb[q] = convb[lc0 + q];
                    }
                    float r0[8], r1[8], r2[8];
                    raw(j0 - 3, r0);
                    raw(j0 - 2, r1);
                    raw(j0 - 1, r2);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float r3[8];
                        if (j0 + i < cnt) {
                            raw(j0 + i, r3);
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) r3[q] = 0.0f;
                        }
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            float acc = bb[q];
                            acc = fmaf(w0[q], r0[q], acc);
                            acc = fmaf(w1[q], r1[q], acc);
                            acc = fmaf(w2[q], r2[q], acc);
                            acc = fmaf(w3[q], r3[q], acc);
                            o[i][q] = (j0 + i < cnt) ? silu_f(acc) : 0.0f;
                            r0[q] = r1[q]; r1[q] = r2[q]; r2[q] = r3[q];
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        if (j0 + i < cnt) {
                            raw(j0 + i, o[i]);
                        } else {
#pragma unroll
                            for (int q = 0; q < 8; ++q) o[i][q] = 0.0f;
                        }
                    }
                }
            }
            // store 8 rows (slots) x one 16-byte piece
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t rr = j0 + i;
                if (g < kP / 8) {
                    *reinterpret_cast<uint4 *>(sm + kOffX + tc::sw128(rr, g)) = pack8(o[i]);
                    float xw[8];
                    const float wj = wgt[rr];
#pragma unroll
                    for (int q = 0; q < 8; ++q) xw[q] = o[i][q] * wj;
                    *reinterpret_cast<uint4 *>(sm + kOffXw + tc::sw128(rr, g)) = pack8(xw);
                } else {
                    const int n0 = lc0 - kP;                       // 0..255 over B then C
                    const uint32_t base = n0 < kN ? kOffB : kOffC;
                    const int nn = n0 < kN ? n0 : n0 - kN;         // 0..127
                    *reinterpret_cast<uint4 *>(sm + base + (nn >> 6) * 16384 +
                                               tc::sw128(rr, (nn & 63) >> 3)) = pack8(o[i]);
                }
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();

        // ---- C: G = C B^T
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t idG = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
            for (int ks = 0; ks < kN / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kColG, tc::smem_desc(sbase + kOffC + koff, 16, 1024),
                             tc::smem_desc(sbase + kOffB + koff, 16, 1024), idG, ks > 0);
            }
            tc::mma_commit(mbar);
        }
        ok = tc::mbar_wait_bounded(mbar, phase, kWaitCycles);
        phase ^= 1;
        if (!__syncthreads_and(ok)) break;
        tc::fence_after_sync();

        // ---- D: M = mask(G * exp(c_t - c_s) * dt_s) -> bf16 tile [t][s]
        {
            const float ct = cum[row];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const int jb = 2 * half + jj;       // 32-column block of s
                float m[32];
                if (jb <= (warp & 3)) {             // warp-uniform: block has s <= t
                    float gv[32];
                    tc::tmem_ld32(tmem + lane_base + kColG + 32 * jb, gv);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int s = 32 * jb + i;
                        const float e = __expf(fminf(ct - cum[s], 0.0f));
                        m[i] = (s <= row) ? gv[i] * e * dts[s] : 0.0f;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) m[i] = 0.0f;
                }
#pragma unroll
                for (int pc = 0; pc < 4; ++pc)
                    *reinterpret_cast<uint4 *>(sm + kOffM + (jb >> 1) * 16384 +
                                               tc::sw128(row, 4 * (jb & 1) + pc)) = pack8(m + 8 * pc);
            }
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();

        // ---- E: Y_diag = M X, Y_off = C S_in^T, dS^T = B^T (wX)
        if (tid == 0) {
            tc::fence_after_sync();
            constexpr uint32_t idY = tc::idesc_bf16(128, 64, 0, 1);
            constexpr uint32_t idS = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < kQ / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kColYd, tc::smem_desc(sbase + kOffM + koff, 16, 1024),
                             tc::smem_desc(sbase + kOffX + ks * 2048, 1024, 1024), idY, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < kN / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kColYo, tc::smem_desc(sbase + kOffC + koff, 16, 1024),
                             tc::smem_desc(sbase + kOffS + ks * 2048, 1024, 1024), idY, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < kQ / 16; ++ks) {
                tc::mma_bf16(tmem + kColDS, tc::smem_desc(sbase + kOffB + ks * 2048, 16384, 1024),
                             tc::smem_desc(sbase + kOffXw + ks * 2048, 1024, 1024), idS, ks > 0);
            }
            tc::mma_commit(mbar);
        }
        ok = tc::mbar_wait_bounded(mbar, phase, kWaitCycles);
        phase ^= 1;
        if (!__syncthreads_and(ok)) break;
        tc::fence_after_sync();

        // ---- F: state update and output
        {
            float ds[32];
            tc::tmem_ld32(tmem + lane_base + kColDS + 32 * half, ds);
            const float a_last = __expf(cum_last);
#pragma unroll
            for (int q = 0; q < 32; ++q) S[q] = fmaf(a_last, S[q], ds[q]);
        }
        float yv[32];
        {
            float yd[32], yo[32];
            tc::tmem_ld32(tmem + lane_base + kColYd + 32 * half, yd);
            tc::tmem_ld32(tmem + lane_base + kColYo + 32 * half, yo);
            const float et = __expf(cum[row]);
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                float xv[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + kOffX + tc::sw128(row, 4 * half + pc)), xv);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int i = 8 * pc + q;
                    yv[i] = fmaf(et, yo[i], yd[i]) + Dh * xv[q];
                }
            }
        }
        tc::fence_before_sync();
        store_state_bf16();   // the Y_off MMA that read the old copy has completed

        // forward + reverse sum through the per-chunk handshake
        int *fl = p.flags + (((size_t)b * H + h) * p.nchunks + c) * 2;
        if (tid == 0) *flag_slot = atomicAdd(fl, 1);
        __syncthreads();
        const bool first = *flag_slot == 0;
        const bool valid = row < cnt;
        const int tok = rev ? t0 + cnt - 1 - row : t0 + row;
        __nv_bfloat16 *yrow = p.y + ((size_t)b * L + tok) * ((size_t)H * kP) + h * kP + 32 * half;
        if (first) {
            if (valid) {
#pragma unroll
                for (int pc = 0; pc < 4; ++pc)
                    reinterpret_cast<uint4 *>(yrow)[pc] = pack8(yv + 8 * pc);
            }
            __threadfence();
            __syncthreads();
            if (tid == 0) atomicExch(fl + 1, 1);
        } else {
            if (tid == 0) {
                bool ready = ld_acquire(fl + 1) != 0;
                if (!ready) {
                    const long long w0 = clock64();
                    while (!(ready = ld_acquire(fl + 1) != 0)) {
                        if (clock64() - w0 > kWaitCycles) break;
                    }
                }
                if (!ready) record_error(p.status, kStatusTimeout);
            }
            __syncthreads();
            __threadfence();
            if (valid) {
#pragma unroll
                for (int pc = 0; pc < 4; ++pc) {
                    float prev[8];
                    unpack8(__ldcg(reinterpret_cast<const uint4 *>(yrow) + pc), prev);
#pragma unroll
                    for (int q = 0; q < 8; ++q) prev[q] += yv[8 * pc + q];
                    reinterpret_cast<uint4 *>(yrow)[pc] = pack8(prev);
                }
            }
            __syncthreads();
            if (tid == 0) {
                fl[0] = 0;   // leave the workspace zeroed for the next call
                fl[1] = 0;
            }
        }
    }

    if (ok && !rev && p.fin) {
#pragma unroll
        for (int q = 0; q < 32; ++q) p.fin[sidx + (size_t)(32 * half + q) * kN + row] = S[q];
    }
    if (!ok && tid == 0) record_error(p.status, kStatusTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

bool tc_path_supported(const bimamba_dims &d)
{
    return d.dtype == BIMAMBA_BF16 && d.headdim == kP && d.d_state == kN && d.ngroups == 1 &&
           d.d_conv == 4 && d.len > 0;
}

size_t tc_workspace_bytes(const bimamba_dims &d)
{
    const size_t nchunks = ((size_t)d.len + kQ - 1) / kQ;
    const size_t bytes = (size_t)d.batch * d.heads * nchunks * 2 * sizeof(int);
    return (bytes + 255) & ~(size_t)255;
}

cudaError_t launch_ssd_tc(const Problem &pr, cudaStream_t stream)
{
    const bimamba_dims &d = pr.dims;
    TcParams p;
    p.xbc = static_cast<const __nv_bfloat16 *>(pr.xbc);
    p.dt = static_cast<const __nv_bfloat16 *>(pr.dt);
    p.A = pr.A;
    p.D = pr.D;
    p.conv_w = pr.conv_w;
    p.conv_b = pr.conv_b;
    p.tail = static_cast<const __nv_bfloat16 *>(pr.tail);
    p.init = pr.init;
    p.fin = pr.fin;
    p.y = static_cast<__nv_bfloat16 *>(pr.y);
    p.flags = static_cast<int *>(pr.workspace);
    p.status = pr.status;
    p.len = d.len;
    p.H = d.heads;
    p.ch = d.heads * d.headdim + 2 * d.ngroups * d.d_state;
    p.nchunks = (d.len + kQ - 1) / kQ;
    cudaError_t ea = cudaFuncSetAttribute(ssd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          (int)kSmemBytes);
    if (ea != cudaSuccess) return ea;
    ssd_tc_kernel<<<dim3(2 * d.heads, d.batch), kThreads, kSmemBytes, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

}  // namespace bimamba
