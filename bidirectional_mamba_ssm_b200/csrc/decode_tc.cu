// decode_tc.cu -- cached block decode for block diffusion on the sm_100a
// tensor cores, for active blocks of at most 64 tokens.
//
// Operation ("Fixed state, long reach: constant-size caches in large-scale
// block diffusion", abstract and section 1: a finished prefix is cached as
// the forward SSM state, O(1) in the context length, plus the conv history;
// the reverse scan is restricted to the active block; with the Mamba-2
// recurrence of "DiffuMamba: High-Throughput Diffusion LMs with Mamba
// Backbone", technical summaries section 2, forward and reverse streams
// added):
//   forward : h_{-1} = S_in (cached), conv history = the tail's newest 3
//             tokens; y_f[t] = sum_{s<=t} M_f[t,s] x_f[s] + exp(c_t) C_f[t] S_in^T
//   reverse : zero state, zero padding past the block end, in walk order
//             j <-> token len-1-j; y_r = M_r x_r
//   y = y_f + y_r;  commit: S_out = exp(c_last) S_in + B_f^T (w o X_f)
// with M[t,s] = (C_t . B_s) exp(c_t - c_s) dt_s (s < t), (C_t . B_t) dt_t + D
// (s = t), c = inclusive prefix sums of dt*A in walk order.
//
// Two kernels:
//  * decode_prep_kernel, one CTA per stream: conv+SiLU of the block's B and
//    C channels for both directions, stacked as [forward; reverse] 128-row
//    tiles; G = C B^T for both at once (one 128 x 128 x 128 tcgen05 product
//    whose diagonal 64 x 64 blocks are G_f and G_r); writes G (fp32) and the
//    forward C and B tiles as ready-made shared-memory images.
//  * decode_tc_kernel, one CTA per (stream, head), both directions: the
//    cached state (fp32 -> bf16, K-major), the forward C/B images by one bulk
//    copy, the conv of the head's x for both directions (stacked rows
//    [forward slots; reverse walk slots]), M for both directions as one
//    block-diagonal 128 x 128 operand in tensor memory, then
//      Yd = M . [X_f; X_r]          (A in TMEM, 128 x 64 x 128)
//      Yo = C_f . S_in^T            (128 x 64 x 128; rows 64..127 unused)
//      dS^T = B_f^T . (w o X_f)     (commit only)
//    and the sum of the two streams through a shared-memory staging tile.
//    Each CTA uses 256 tensor-memory columns and ~76 KB of shared memory, so
//    two CTAs share an SM and one's state load overlaps the other's math.
//
// The state pool form (bimamba_block_decode_pool) reads each batch row's
// state and conv tail from a pool slot and commits per row.
#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace bimamba {

namespace {

constexpr int kDQ = 64;        // block slots per direction
constexpr int kDP = 64;        // headdim
constexpr int kDN = 128;       // d_state
constexpr int kDThreads = 256;
constexpr long long kDWait = 4000000000LL;   // ~2 s at 1.9 GHz

// decode_prep_kernel shared memory: [C_f; C_r] and [B_f; B_r], each K-major
// with 128-byte swizzle, two 64-channel atoms of 128 rows (16 KB each)
constexpr uint32_t kPOffC = 0;
constexpr uint32_t kPOffB = 32768;
constexpr uint32_t kPOffMbar = 65536;
constexpr uint32_t kPOffTmem = kPOffMbar + 8;
constexpr uint32_t kPSmem = kPOffTmem + 8 + 1024;

// per-stream prep record in the workspace: G_f, G_r (fp32 64 x 64 each),
// then the forward C and B shared-memory images (2 atoms of 64 rows x 128 B each)
constexpr size_t kPrepG = 2 * kDQ * kDQ * sizeof(float);   // 32 KB
constexpr size_t kPrepImg = 4 * kDQ * 128;                  // 32 KB: C atom 0, C atom 1, B atom 0, B atom 1
constexpr size_t kPrepBytes = kPrepG + kPrepImg;

// decode_tc_kernel shared memory
constexpr uint32_t kDOffS = 0;          // S_in bf16 K-major [2 atoms][64 p][128 B]; then fp32 staging
constexpr uint32_t kDOffC = 16384;      // C_f image (the Yo operand reads 128 rows: C_f then B_f)
constexpr uint32_t kDOffB = 24576 + 8192;   // B_f image
constexpr uint32_t kDOffX = 49152;      // [X_f; X_r] MN-major [128 slots][64 p]
constexpr uint32_t kDOffXw = 65536;     // w o X_f [64 slots][64 p]
// the cached fp32 state [64 p][128 n], landed by one bulk copy where X and
// wX go later (it is converted to the bf16 tile before the conv writes X)
constexpr uint32_t kDOffSf = kDOffX;
// raw x rows, rho = token rho - 3, 128 bytes each with the 128-byte swizzle
// keyed on (rho + 5) & 7: the 3 conv-tail rows, then the TMA box of the
// block's 64 tokens (1024-aligned; rows past the block end read zeros)
constexpr uint32_t kDOffRawBox = 82944;
constexpr uint32_t kDOffRaw = kDOffRawBox - 3 * 128;
constexpr uint32_t kDOffCum = kDOffRawBox + kDQ * 128;   // f32 cf[64], cr[64], dtf[64], dtr[64]
constexpr uint32_t kDOffF8 = kDOffCum + 1024;     // f32 f8f[64], f8r[64]: exp(c_R - c_s) dt_s, R = s | 7
constexpr uint32_t kDOffConvW = kDOffF8 + 512;     // float4[64]
constexpr uint32_t kDOffConvB = kDOffConvW + 1024; // f32[64]
constexpr uint32_t kDOffMbar = kDOffConvB + 256;   // 2 mbarriers
constexpr uint32_t kDOffTmem = kDOffMbar + 16;
constexpr uint32_t kDSmem = kDOffTmem + 16 + 1024;
static_assert(kDOffB == kDOffC + 16384, "C_f and B_f images are one contiguous copy");
static_assert(kDOffSf + kDP * kDN * 4 <= kDOffRaw && kDOffRawBox % 1024 == 0, "decode shared-memory map");

constexpr uint32_t kDColM = 0, kDColYd = 64, kDColYo = 128, kDColS = 192;

__device__ __forceinline__ void unpack8f(uint4 r, float (&v)[8])
{
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ uint4 pack8f(const float *v)
{
    uint4 r;
    r.x = tc::pack_bf16x2(v[0], v[1]);
    r.y = tc::pack_bf16x2(v[2], v[3]);
    r.z = tc::pack_bf16x2(v[4], v[5]);
    r.w = tc::pack_bf16x2(v[6], v[7]);
    return r;
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to shared memory, completion counted on `mbar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t mbar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        :: "r"(dst), "l"(src), "r"(bytes), "r"(mbar) : "memory");
}

}  // namespace

// One CTA per stream.  Thread (channel group g of 8, row group rg of 16
// stacked rows): rows 0..63 forward slots (token j; the tail supplies the
// 3 tokens before the block), rows 64..127 reverse walk slots (token
// len-1-j; zeros past the block end).  Slots past len are zero.
__global__ void __launch_bounds__(kDThreads, 1)
decode_prep_kernel(const __nv_bfloat16 *__restrict__ xbc, const __nv_bfloat16 *__restrict__ tail,
                   const int *__restrict__ slots, int pool, const float *__restrict__ conv_w,
                   const float *__restrict__ conv_b, uint8_t *__restrict__ prep, int len, int ch,
                   int cbase, int *status)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5;
    const int s = blockIdx.x;
    // the decode kernel may start now: it loads its inputs that do not come
    // from here, then waits for this grid (griddepcontrol.wait) before
    // reading the records
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int slot = slots ? slots[s] : s;
    if (slot < 0 || slot >= pool) return;   // uniform: the decode kernel records the error
    const uint32_t mb = sbase + kPOffMbar;
    if (warp == 0) tc::tmem_alloc(sbase + kPOffTmem, 128);
    if (tid == 0) tc::mbar_init(mb, 1);

    {
        const int g = tid & 31;            // channels 8g .. 8g+7 of B|C
        const int rg = tid >> 5;           // stacked rows 16 rg .. 16 rg + 15
        const bool rev = rg >= 4;
        const int j0 = 16 * (rg & 3);
        const int c = cbase + 8 * g;
        const __nv_bfloat16 *xb = xbc + (size_t)s * len * ch + c;
        const __nv_bfloat16 *tb = tail + (size_t)slot * 4 * ch + c;
        float w0[8], w1[8], w2[8], w3[8], bb[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 t4 = *reinterpret_cast<const float4 *>(conv_w + (size_t)(c + q) * 4);
            w0[q] = t4.x; w1[q] = t4.y; w2[q] = t4.z; w3[q] = t4.w;
            bb[q] = conv_b ? conv_b[c + q] : 0.0f;
        }
        // the 19 raw rows of this thread's 16 slots (3 before), loaded first
        uint4 rw[19];
#pragma unroll
        for (int i = 0; i < 19; ++i) {
            const int j = j0 + i - 3;
            const int tok = rev ? len - 1 - j : j;
            rw[i] = (tok >= 0 && tok < len) ? __ldg(reinterpret_cast<const uint4 *>(xb + (size_t)tok * ch))
                    : (!rev && tok < 0 && tok >= -4) ? __ldg(reinterpret_cast<const uint4 *>(tb + (size_t)(4 + tok) * ch))
                                                      : make_uint4(0, 0, 0, 0);
        }
        const int cc = (8 * g) & 127;                    // channel within B or C
        uint8_t *tile = sm + ((8 * g < 128) ? kPOffB : kPOffC) + (cc >> 6) * 16384;
        const int piece = (cc & 63) >> 3;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int j = j0 + i;
            float r0[8], r1[8], r2[8], r3[8], o[8];
            unpack8f(rw[i], r0);
            unpack8f(rw[i + 1], r1);
            unpack8f(rw[i + 2], r2);
            unpack8f(rw[i + 3], r3);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                float acc = bb[q];
                acc = fmaf(w0[q], r0[q], acc);
                acc = fmaf(w1[q], r1[q], acc);
                acc = fmaf(w2[q], r2[q], acc);
                acc = fmaf(w3[q], r3[q], acc);
                o[q] = (j < len) ? tc::silu_tanh(acc) : 0.0f;
            }
            const int row = 16 * rg + i;
            *reinterpret_cast<uint4 *>(tile + tc::sw128(row, piece)) = pack8f(o);
        }
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kPOffTmem);
    bool ok = true;
    if (tid == 0) {
        const uint64_t dC = tc::smem_desc(sbase + kPOffC, 16, 1024);
        const uint64_t dB = tc::smem_desc(sbase + kPOffB, 16, 1024);
        constexpr uint32_t idG = tc::idesc_bf16(128, 128, 0, 0);
#pragma unroll
        for (int ks = 0; ks < kDN / 16; ++ks) {
            const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
            tc::mma_bf16(tmem, tc::desc_add(dC, koff), tc::desc_add(dB, koff), idG, ks > 0);
        }
        tc::mma_commit(mb);
        ok = tc::mbar_wait_bounded(mb, 0, kDWait);
        if (!ok) record_error(status, kStatusTimeout);
    }
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    uint8_t *rec = prep + (size_t)s * kPrepBytes;
    if (ok && warp < 4) {
        // G_f = rows 0..63 x cols 0..63, G_r = rows 64..127 x cols 64..127
        const int r = tid;                    // TMEM lane
        const int d = r >> 6, t = r & 63;
        float g[32];
        float *gout = reinterpret_cast<float *>(rec) + ((size_t)d * kDQ + t) * kDQ;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tc::tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + 64 * d + 32 * half, g);
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(gout + 32 * half + i) = make_float4(g[i], g[i + 1], g[i + 2], g[i + 3]);
        }
    }
    // the forward rows (0..63) of each atom of C and B, as shared-memory images
    {
        const uint4 *srcC = reinterpret_cast<const uint4 *>(sm + kPOffC);
        const uint4 *srcB = reinterpret_cast<const uint4 *>(sm + kPOffB);
        uint4 *dst = reinterpret_cast<uint4 *>(rec + kPrepG);
        for (int i = tid; i < 4 * 512; i += kDThreads) {   // 4 images of 8 KB (512 x 16 B)
            const int img = i >> 9, e = i & 511;
            const uint4 *src = (img < 2 ? srcC : srcB) + (img & 1) * 1024 + e;
            dst[i] = *src;
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 128);
}

struct DecodeParams {
    int pool;                     // pool size (slots are checked against it)
    const __nv_bfloat16 *xbc;     // (S, len, ch) raw block
    const __nv_bfloat16 *dt;      // (S, len, H)
    const float *A, *D, *conv_w, *conv_b;
    const float *state;           // (pool, H, P, N): the cached forward states
    const __nv_bfloat16 *tail;    // (pool, 4, ch)
    const int *slots;             // (S) pool slot of each batch row, or null (row s = slot s)
    const int *commit;            // (S) commit flags, or null (commit every row when state_out)
    float *state_out;             // (pool, H, P, N) or null
    __nv_bfloat16 *y;             // (S, len, H*P)
    const uint8_t *prep;          // per-stream prep records
    int *status;
    int len, H, ch;
};

// One CTA per (stream, head): both directions of one head over the block.
__global__ void __launch_bounds__(kDThreads, 2)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_x, const DecodeParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, s = blockIdx.y;
    const int H = p.H, len = p.len, ch = p.ch;
    const int slot = p.slots ? p.slots[s] : s;
    if (slot < 0 || slot >= p.pool) {   // uniform over the CTA: nothing allocated yet
        if (tid == 0 && h == 0) record_error(p.status, kStatusBadSlot);
        return;
    }
    const bool do_commit = p.state_out && (!p.commit || p.commit[s] != 0);
    float *cf = reinterpret_cast<float *>(sm + kDOffCum);
    float *cr = cf + 64, *dtf = cf + 128, *dtr = cf + 192;
    float *f8f = reinterpret_cast<float *>(sm + kDOffF8), *f8r = f8f + 64;
    float4 *convw = reinterpret_cast<float4 *>(sm + kDOffConvW);
    float *convb = reinterpret_cast<float *>(sm + kDOffConvB);
    const uint32_t mb_ld = sbase + kDOffMbar, mb_mma = mb_ld + 8;
    const uint8_t *rec = p.prep + (size_t)s * kPrepBytes;
    const float *state = p.state + ((size_t)slot * H + h) * kDP * kDN;

    // Every global input is requested up front, so that one memory latency
    // covers them all: the C_f / B_f images, the cached state and the
    // block's raw x rows by bulk / TMA copies onto one mbarrier, the conv
    // tail and G rows by plain loads.
    if (warp == 0) tc::tmem_alloc(sbase + kDOffTmem, 256);
    if (tid == 0) {
        tc::mbar_init(mb_ld, 1);
        tc::mbar_init(mb_mma, 1);
        tc::prefetch_tmap(&tm_x);
        tc::mbar_expect_tx(mb_ld, 32768 + kDP * kDN * 4 + kDQ * 128);
        bulk_g2s(sbase + kDOffSf, state, kDP * kDN * 4, mb_ld);        // the cached state
        tc::tma_load_3d(sbase + kDOffRawBox, &tm_x, h * kDP, 0, s, mb_ld);   // tokens 0..63 (zeros past len)
        // the prep records of this step (C_f and B_f images) once their grid is done
        asm volatile("griddepcontrol.wait;" ::: "memory");
        bulk_g2s(sbase + kDOffC, rec + kPrepG, 32768, mb_ld);
    }
    if (tid >= 64 && tid < 64 + 24) {
        // conv tail: the 3 newest tokens before the block, raw rows 0..2
        const int e = tid - 64, rr = e >> 3, c = e & 7;
        const uint4 v = *reinterpret_cast<const uint4 *>(p.tail + ((size_t)slot * 4 + 1 + rr) * ch + h * kDP + 8 * c);
        *reinterpret_cast<uint4 *>(sm + kDOffRaw + rr * 128 + ((c ^ ((rr + 5) & 7)) << 4)) = v;
    }
    if (tid < kDP) {
        const int c = h * kDP + tid;
        const float4 w = *reinterpret_cast<const float4 *>(p.conv_w + (size_t)c * 4);
        convw[tid] = make_float4(0.5f * w.x, 0.5f * w.y, 0.5f * w.z, 0.5f * w.w);   // halved (see the conv)
        convb[tid] = p.conv_b ? 0.5f * p.conv_b[c] : 0.0f;
    }
    if (warp == 7) {
        // dt of the head, prefix sums of dt*A in log2 units: forward in token
        // order, reverse in walk order (token len-1-j)
        const float Al = p.A[h] * 1.4426950408889634f;
        float d[2], e[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int j = 2 * lane + i;
            d[i] = j < len ? __bfloat162float(p.dt[((size_t)s * len + j) * H + h]) : 0.0f;
            const int jr = len - 1 - j;
            e[i] = j < len ? __bfloat162float(p.dt[((size_t)s * len + jr) * H + h]) : 0.0f;
        }
        float af0 = d[0] * Al, af1 = fmaf(d[1], Al, af0);
        float ar0 = e[0] * Al, ar1 = fmaf(e[1], Al, ar0);
        float runf = af1, runr = ar1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const float vf = __shfl_up_sync(0xffffffffu, runf, o);
            const float vr = __shfl_up_sync(0xffffffffu, runr, o);
            if (lane >= o) {
                runf += vf;
                runr += vr;
            }
        }
        const float xf = runf - af1, xr = runr - ar1;
        cf[2 * lane] = xf + af0;
        cf[2 * lane + 1] = xf + af1;
        cr[2 * lane] = xr + ar0;
        cr[2 * lane + 1] = xr + ar1;
        dtf[2 * lane] = d[0];
        dtf[2 * lane + 1] = d[1];
        dtr[2 * lane] = e[0];
        dtr[2 * lane + 1] = e[1];
        __syncwarp();
        // per-slot factors of the 8-slot groups (from the sums the other lanes wrote)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int j = 2 * lane + i;
            f8f[j] = tc::exp2_approx(cf[j | 7] - cf[j]) * d[i];
            f8r[j] = tc::exp2_approx(cr[j | 7] - cr[j]) * e[i];
        }
    }
    // thread (r, half): stacked row r (TMEM lane) -- direction d = r >> 6,
    // walk slot t = r & 63 -- and the half of the 64 channels / slots it owns
    const int r = tid & 127, half = tid >> 7;
    const int d = r >> 6, t = r & 63;
    // this thread's G row (L2-resident prep record), loaded while the copies fly
    float4 grow[8];
    asm volatile("griddepcontrol.wait;" ::: "memory");   // (the prep grid's records are written)
    {
        const float4 *grow4 = reinterpret_cast<const float4 *>(
            reinterpret_cast<const float *>(rec) + ((size_t)d * kDQ + t) * kDQ + 32 * half);
#pragma unroll
        for (int i = 0; i < 8; ++i) grow[i] = __ldg(grow4 + i);
    }
    tc::fence_before_sync();
    __syncthreads();   // mbarrier initialised; taps, prefix sums and tail rows written
    bool ok = tc::mbar_wait_bounded(mb_ld, 0, kDWait);
    if (!ok && tid == 0) record_error(p.status, kStatusTimeout);
    ok = __syncthreads_and(ok);
    if (ok) {
        // the cached state S[p][n] (fp32, shared) -> bf16 K-major tile (N = p
        // rows, K = n; atom n / 64).  Thread (row pr, quad pc) of step i: n =
        // 4 pc .. 4 pc + 3 of each atom, so that a half-warp reads 256
        // contiguous bytes per load (no bank conflicts) and writes one row of
        // each atom in 8-byte halves of its 16-byte pieces
        const float *sf = reinterpret_cast<const float *>(sm + kDOffSf);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = tid + kDThreads * i;
            const int pr = e >> 4, pc = e & 15;
            const float4 a = *reinterpret_cast<const float4 *>(sf + pr * kDN + 4 * pc);
            const float4 b4 = *reinterpret_cast<const float4 *>(sf + pr * kDN + 64 + 4 * pc);
            const uint32_t off = tc::sw128(pr, pc >> 1) + 8 * (pc & 1);
            *reinterpret_cast<uint2 *>(sm + kDOffS + off) =
                make_uint2(tc::pack_bf16x2(a.x, a.y), tc::pack_bf16x2(a.z, a.w));
            *reinterpret_cast<uint2 *>(sm + kDOffS + 8192 + off) =
                make_uint2(tc::pack_bf16x2(b4.x, b4.y), tc::pack_bf16x2(b4.z, b4.w));
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kDOffTmem);

    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    const float *cdir = d ? cr : cf;
    const float *dtdir = d ? dtr : dtf;

    // ---- conv+SiLU of the head's x into [X_f; X_r], and w o X_f for the
    // commit, from the raw rows in shared memory.  Thread: channel quad cq
    // (channels 4cq .. 4cq+3) x 8 stacked rows 8g .. 8g+7 (direction
    // g >> 3), in packed fp32 pairs with halved taps and bias: SiLU(a) =
    // h + h tanh(h), h = a / 2.  Raw row of slot t's tap j: t + j forward,
    // len + 5 - t - j reverse (token len-1-t, mirrored taps); tokens past
    // the block end read zeros.
    if (ok) {
        const int cq = tid & 15, g = tid >> 4;
        const int dg = g >> 3, t0 = 8 * (g & 7);
        uint2 rr[11];
#pragma unroll
        for (int i = 0; i < 11; ++i) {
            const int rho = dg ? len + 5 - t0 - i : t0 + i;
            const int chunk = cq >> 1;
            rr[i] = (rho >= 0 && rho < len + 3)
                        ? *reinterpret_cast<const uint2 *>(sm + kDOffRaw + rho * 128 +
                                                           ((chunk ^ ((rho + 5) & 7)) << 4) + 8 * (cq & 1))
                        : make_uint2(0u, 0u);
        }
        float4 wq[4];
        float bq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            wq[q] = convw[4 * cq + q];
            bq[q] = convb[4 * cq + q];
        }
        const float2 wa0 = make_float2(wq[0].x, wq[1].x), wa1 = make_float2(wq[0].y, wq[1].y);
        const float2 wa2 = make_float2(wq[0].z, wq[1].z), wa3 = make_float2(wq[0].w, wq[1].w);
        const float2 wb0 = make_float2(wq[2].x, wq[3].x), wb1 = make_float2(wq[2].y, wq[3].y);
        const float2 wb2 = make_float2(wq[2].z, wq[3].z), wb3 = make_float2(wq[2].w, wq[3].w);
        const float2 ba = make_float2(bq[0], bq[1]), bb = make_float2(bq[2], bq[3]);
        auto up = [](uint32_t v) { return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v)); };
        float2 a0 = up(rr[0].x), a1 = up(rr[1].x), a2 = up(rr[2].x);
        float2 b0 = up(rr[0].y), b1 = up(rr[1].y), b2 = up(rr[2].y);
        const bool commit_rows = do_commit && dg == 0;
        const float c_last = cf[len - 1];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int tt = t0 + i;
            const float2 a3 = up(rr[i + 3].x), b3 = up(rr[i + 3].y);
            float2 ha = tc::fma2(wa0, a0, ba);
            float2 hb = tc::fma2(wb0, b0, bb);
            ha = tc::fma2(wa1, a1, ha);
            hb = tc::fma2(wb1, b1, hb);
            ha = tc::fma2(wa2, a2, ha);
            hb = tc::fma2(wb2, b2, hb);
            ha = tc::fma2(wa3, a3, ha);
            hb = tc::fma2(wb3, b3, hb);
            float th[4];
            asm("tanh.approx.f32 %0, %1;" : "=f"(th[0]) : "f"(ha.x));
            asm("tanh.approx.f32 %0, %1;" : "=f"(th[1]) : "f"(ha.y));
            asm("tanh.approx.f32 %0, %1;" : "=f"(th[2]) : "f"(hb.x));
            asm("tanh.approx.f32 %0, %1;" : "=f"(th[3]) : "f"(hb.y));
            float2 oa = tc::fma2(ha, make_float2(th[0], th[1]), ha);
            float2 ob = tc::fma2(hb, make_float2(th[2], th[3]), hb);
            if (tt >= len) {
                oa = make_float2(0.0f, 0.0f);
                ob = oa;
            }
            const uint32_t off = tc::sw128(8 * g + i, cq >> 1) + 8 * (cq & 1);
            *reinterpret_cast<uint2 *>(sm + kDOffX + off) =
                make_uint2(tc::pack_bf16x2(oa.x, oa.y), tc::pack_bf16x2(ob.x, ob.y));
            if (commit_rows) {
                const float wc = tt < len ? tc::exp2_approx(c_last - cf[tt]) * dtf[tt] : 0.0f;
                const float2 w2 = make_float2(wc, wc);
                const float2 xa = tc::mul2(oa, w2), xb = tc::mul2(ob, w2);
                *reinterpret_cast<uint2 *>(sm + kDOffXw + off) =
                    make_uint2(tc::pack_bf16x2(xa.x, xa.y), tc::pack_bf16x2(xb.x, xb.y));
            }
            a0 = a1; a1 = a2; a2 = a3;
            b0 = b1; b1 = b2; b2 = b3;
        }
    }
    // ---- M: row r holds its direction's 64 K columns [64 d, 64 d + 64)
    // (this thread: slots 32 half .. 32 half + 31) and zeros in the other
    // direction's; D on the diagonal
    if (ok) {
        const float Dh = p.D[h];
        float g[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float4 v = grow[i];
            g[4 * i] = v.x; g[4 * i + 1] = v.y; g[4 * i + 2] = v.z; g[4 * i + 3] = v.w;
        }
        // groups of 8 slots: exp(c_t - c_s) dt_s = exp(c_t - c_R) f8[s], R the group's
        // last slot.  With the group's own decay at most 2^60 neither factor
        // overflows where the element is kept (s <= t); else one exponential
        // per element, each <= 1.  (The direction is uniform over a warp.)
        const float ct = cdir[t];
        const float *f8dir = d ? f8r : f8f;
        uint32_t packed[16], zero[16];
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
            const int sb = 32 * half + 8 * g8;
            float m[8];
            if (cdir[sb] - cdir[sb + 7] <= 60.0f) {
                const float et = tc::exp2_approx(ct - cdir[sb + 7]);
#pragma unroll
                for (int e = 0; e < 8; ++e) m[e] = g[8 * g8 + e] * et * f8dir[sb + e];
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    m[e] = g[8 * g8 + e] * tc::exp2_approx(fminf(ct - cdir[sb + e], 0.0f)) * dtdir[sb + e];
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int sl = sb + e;
                const float me = (sl == t) ? fmaf(g[8 * g8 + e], dtdir[t], Dh) : m[e];
                m[e] = (sl <= t && t < len) ? me : 0.0f;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                packed[4 * g8 + q] = tc::pack_bf16x2(m[2 * q], m[2 * q + 1]);
                zero[4 * g8 + q] = 0u;
            }
        }
        tc::tmem_st16(tmem + lane_base + kDColM + 32 * d + 16 * half, packed);
        tc::tmem_st16(tmem + lane_base + kDColM + 32 * (1 - d) + 16 * half, zero);
    }
    tc::fence_proxy_async();
    tc::fence_before_sync();
    __syncthreads();
    if (ok && tid == 0) {
        tc::fence_after_sync();
        {
            const uint64_t dX = tc::smem_desc(sbase + kDOffX, 1024, 1024);     // MN-major, N = 64
            const uint64_t dC = tc::smem_desc(sbase + kDOffC, 16, 1024);       // K-major A
            const uint64_t dS = tc::smem_desc(sbase + kDOffS, 16, 1024);       // K-major B (N = p)
            const uint64_t dBmn = tc::smem_desc(sbase + kDOffB, 8192, 1024);   // MN-major A (M = n)
            const uint64_t dXw = tc::smem_desc(sbase + kDOffXw, 1024, 1024);   // MN-major B
            constexpr uint32_t idYd = tc::idesc_bf16(128, 64, 0, 1);
            constexpr uint32_t idYo = tc::idesc_bf16(128, 64, 0, 0);
            constexpr uint32_t idS = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < 2 * kDQ / 16; ++ks)
                tc::mma_bf16_tmemA(tmem + kDColYd, tmem + kDColM + 8 * ks, tc::desc_add(dX, ks * 2048), idYd,
                                   ks > 0);
#pragma unroll
            for (int ks = 0; ks < kDN / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 8192 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kDColYo, tc::desc_add(dC, koff), tc::desc_add(dS, koff), idYo, ks > 0);
            }
            if (do_commit) {
#pragma unroll
                for (int ks = 0; ks < kDQ / 16; ++ks)
                    tc::mma_bf16(tmem + kDColS, tc::desc_add(dBmn, ks * 2048), tc::desc_add(dXw, ks * 2048),
                                 idS, ks > 0);
            }
            tc::mma_commit(mb_mma);
            ok = tc::mbar_wait_bounded(mb_mma, 0, kDWait);
        }
        if (!ok) record_error(p.status, kStatusTimeout);
    }
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    if (ok) {
        // ---- y = forward + reverse.  The reverse rows go to an fp32 staging
        // tile (the state tile's space; token row at tok * 256 bytes, 16-byte
        // chunk q at q ^ (tok & 15)); the forward rows add them and store.
        float yv[32];
        tc::tmem_ld32(tmem + lane_base + kDColYd + 32 * half, yv);
        float *stage = reinterpret_cast<float *>(sm + kDOffS);
        if (d == 1) {
            if (t < len) {
                const int tok = len - 1 - t;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int chunk = 8 * half + q;
                    *reinterpret_cast<float4 *>(stage + tok * 64 + 4 * (chunk ^ (tok & 15))) =
                        make_float4(yv[4 * q], yv[4 * q + 1], yv[4 * q + 2], yv[4 * q + 3]);
                }
            }
        } else {
            float yo[32];
            tc::tmem_ld32(tmem + lane_base + kDColYo + 32 * half, yo);
            const float et = tc::exp2_approx(cf[t]);
#pragma unroll
            for (int i = 0; i < 32; ++i) yv[i] = fmaf(et, yo[i], yv[i]);
        }
        __syncthreads();
        if (d == 0 && t < len) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int chunk = 8 * half + q;
                const float4 v = *reinterpret_cast<const float4 *>(stage + t * 64 + 4 * (chunk ^ (t & 15)));
                yv[4 * q] += v.x;
                yv[4 * q + 1] += v.y;
                yv[4 * q + 2] += v.z;
                yv[4 * q + 3] += v.w;
            }
            uint4 *dst = reinterpret_cast<uint4 *>(p.y + ((size_t)s * len + t) * H * kDP + h * kDP + 32 * half);
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) dst[pc] = pack8f(yv + 8 * pc);
        }
        if (do_commit) {
            // S_out[p][n] = exp(c_last) S_in[p][n] + dS^T[n][p]: thread (lane
            // n = r, half): p = 32 half .. 32 half + 31
            const float a_last = tc::exp2_approx(cf[len - 1]);
            float ds[32];
            tc::tmem_ld32(tmem + lane_base + kDColS + 32 * half, ds);
            float *out = p.state_out + ((size_t)slot * H + h) * kDP * kDN;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const size_t e = (size_t)(32 * half + i) * kDN + r;
                out[e] = fmaf(a_last, state[e], ds[i]);
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

// Conv tails of the committed rows, in place: tail_pool[slot][k] <- (old
// tail | block)[len - 4 + k].  Each thread owns one channel of one row and
// reads its four sources before writing, so the in-place update is safe.
// A slot outside the pool is recorded as an error and skipped.
__global__ void tail_commit_pool_kernel(const __nv_bfloat16 *__restrict__ block,
                                        __nv_bfloat16 *tail_pool, const int *__restrict__ slots,
                                        const int *__restrict__ commit, int pool_size, int len, int ch,
                                        int *status)
{
    const int s = blockIdx.y;
    if (commit && commit[s] == 0) return;
    const int slot = slots ? slots[s] : s;
    if (slot < 0 || slot >= pool_size) {
        if (threadIdx.x == 0 && blockIdx.x == 0) record_error(status, kStatusBadSlot);
        return;
    }
    __nv_bfloat16 *tl = tail_pool + (size_t)slot * 4 * ch;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < ch; c += gridDim.x * blockDim.x) {
        __nv_bfloat16 v[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int pos = len - 4 + k;
            v[k] = pos >= 0 ? block[((size_t)s * len + pos) * ch + c] : tl[(size_t)(4 + pos) * ch + c];
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) tl[(size_t)k * ch + c] = v[k];
    }
}

cudaError_t launch_tail_commit_pool(const void *block, void *tail_pool, const int *slots,
                                    const int *commit, int pool_size, int rows, int len, int ch,
                                    int *status, cudaStream_t stream)
{
    tail_commit_pool_kernel<<<dim3((ch + 255) / 256, rows), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(block), static_cast<__nv_bfloat16 *>(tail_pool), slots,
        commit, pool_size, len, ch, status);
    cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) count_launch();
    return e;
}

bool decode_tc_supported(const bimamba_dims &d)
{
    return d.dtype == BIMAMBA_BF16 && d.headdim == kDP && d.d_state == kDN && d.ngroups == 1 &&
           d.d_conv == 4 && d.len >= 1 && d.len <= kDQ;
}

size_t decode_tc_workspace_bytes(const bimamba_dims &d) { return (size_t)d.batch * kPrepBytes; }

// The block's raw xBC as a 3-D bf16 tensor map (ch, len, streams), read by
// 64-channel x 64-token boxes with the 128-byte swizzle (tokens past len
// read zeros).
static bool make_block_map(CUtensorMap *m, const void *base, int ch, int len, int streams)
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult qr;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &qr) != cudaSuccess ||
            qr != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    const cuuint64_t dims[3] = {(cuuint64_t)ch, (cuuint64_t)len, (cuuint64_t)streams};
    const cuuint64_t strides[2] = {(cuuint64_t)ch * 2, (cuuint64_t)ch * len * 2};
    const cuuint32_t box[3] = {kDP, kDQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_decode_tc(const DecodeProblem &q, cudaStream_t stream)
{
    const bimamba_dims &d = q.dims;
    const int ch = d.heads * d.headdim + 2 * d.ngroups * d.d_state;
    uint8_t *prep = static_cast<uint8_t *>(q.workspace);
    cudaError_t e = cudaFuncSetAttribute(decode_prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kPSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kDSmem);
    if (e != cudaSuccess) return e;
    // the device time of a step: both kernels (the decode kernel overlaps the
    // prep kernel's end through a programmatic dependent launch)
    const TimingEvents ev = timing_events();
    if (ev.start && (e = cudaEventRecord(ev.start, stream)) != cudaSuccess) return e;
    decode_prep_kernel<<<d.batch, kDThreads, kPSmem, stream>>>(
        static_cast<const __nv_bfloat16 *>(q.xbc), static_cast<const __nv_bfloat16 *>(q.tail), q.slots,
        q.pool, q.conv_w, q.conv_b, prep, d.len, ch, d.heads * d.headdim, q.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    DecodeParams p;
    p.xbc = static_cast<const __nv_bfloat16 *>(q.xbc);
    p.dt = static_cast<const __nv_bfloat16 *>(q.dt);
    p.A = q.A;
    p.D = q.D;
    p.conv_w = q.conv_w;
    p.conv_b = q.conv_b;
    p.state = q.state;
    p.tail = static_cast<const __nv_bfloat16 *>(q.tail);
    p.slots = q.slots;
    p.pool = q.pool;
    p.commit = q.commit;
    p.state_out = q.state_out;
    p.y = static_cast<__nv_bfloat16 *>(q.y);
    p.prep = prep;
    p.status = q.status;
    p.len = d.len;
    p.H = d.heads;
    p.ch = ch;
    CUtensorMap tm_x;
    if ((ch * 2) % 16 != 0 || !make_block_map(&tm_x, q.xbc, ch, d.len, d.batch)) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(d.heads, d.batch);
    cfg.blockDim = dim3(kDThreads);
    cfg.dynamicSmemBytes = kDSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, tm_x, p)) != cudaSuccess) return e;
    count_launch();
    if (ev.stop) e = cudaEventRecord(ev.stop, stream);
    return e;
}

}  // namespace bimamba
