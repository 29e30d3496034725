// backward_tc.cu -- the backward of the mixer core on the tensor cores, for
// bf16 activations with headdim 64 and d_state 128 (the 1.3B layer's head
// shape).  Other shapes and fp32 keep the CUDA-core kernels of backward.cu.
//
// The mixer core is the bidirectional Mamba-2 mixer ("DiffuMamba:
// High-Throughput Diffusion LMs with Mamba Backbone", technical summaries
// section 2: forward and reverse streams added; Mamba-2 recurrence h_t =
// exp(dt_t A) h_{t-1} + dt_t x_t B_t^T, y_t = h_t C_t + D x_t), trained with
// the masked-diffusion objective (methodology of the same summaries).  The
// gradients follow the same chunked adjoint as backward.cu, with chunks of
// Q = 128 walk steps.  Per chunk, with c the chunk's prefix sums of dt A,
// W[t,s] = (C_t.B_s) e^{c_t-c_s} dt_s and T[t,s] = (dY_t.x_s) e^{c_t-c_s}
// dt_s for s <= t (walk order), w_s = e^{c_last-c_s} dt_s, S_in the state
// entering the chunk and dS the adjoint of the state leaving it:
//     dX    = W^T dY + D dY + w o (B dS^T)
//     dB    = T^T C + (w o X) dS                (summed over heads)
//     dC    = T B + (e^c o dY) S_in             (summed over heads)
//     dS_in = e^{c_last} dS + (e^c o dY)^T C
// and dt, A through dL/dc of the prefix sums.  Every matrix product above
// (and C B^T, dY X^T, C S_in^T, B dS^T) is a tcgen05 MMA with bf16 operands
// in shared memory and fp32 accumulators in tensor memory; the elementwise
// factors, the sums for dt and A and the epilogues run on the CUDA cores.
//
// Two kernels, one CTA per (head, sequence, direction):
//  * bwd_tc_state_kernel walks the chunks forward and writes the state
//    entering each chunk as a bf16 operand tile S_in^T[n][p] (128-byte
//    swizzle, 16 KB) to the workspace;
//  * bwd_tc_scan_kernel walks them backward with dS in tensor memory.
// The reverse stream walks tokens from the end: a chunk's tiles are loaded
// by TMA in token order (row r = token t0 + r, rows outside the sequence
// read zeros) and row r is walk slot 127 - r.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

namespace bimamba {

namespace {

constexpr int kBQ = 128;   // chunk length (walk slots)
constexpr int kBP = 64;    // headdim
constexpr int kBN = 128;   // d_state
constexpr int kBThreads = 256;   // state pass: tile row r = tid & 127, column half tid >> 7
constexpr int kAThreads = 512;   // adjoint pass: tile row r = tid & 127, column quarter tid >> 7
constexpr long long kBWait = 4000000000LL;   // ~2 s at 1.9 GHz
constexpr float kLog2e = 1.4426950408889634f;
constexpr uint32_t kTileBytes = kBN * kBP * 2;   // one S_in^T tile (16 KB)

struct BwdTcParams {
    const __nv_bfloat16 *dt;   // (batch, len, H)
    const float *A, *D, *init;
    __nv_bfloat16 *states;     // [dir][batch][H][nchunks] S_in^T tiles
    float *dact[2];            // (batch, len, ch) per stream: x part written, B/C parts added
    float *ddt, *dA, *dD, *dinit;
    int *status;
    int batch, len, H, ch, nchunks;
};

__device__ __forceinline__ uint8_t *align1024(uint8_t *p)
{
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// 8 bf16 of a swizzled row piece, unpacked
__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint4 pack8(const float *f)
{
    return make_uint4(tc::pack_bf16x2(f[0], f[1]), tc::pack_bf16x2(f[2], f[3]), tc::pack_bf16x2(f[4], f[5]),
                      tc::pack_bf16x2(f[6], f[7]));
}

// The warp's 32 rows of 32 columns summed per column: v[i] holds column i
// of this lane's row; the result is column `lane`'s sum.  Each step hands
// the half of the columns this lane does not keep to its partner (31
// shuffles in all).
__device__ __forceinline__ float column_sum32(float (&v)[32], int lane)
{
#pragma unroll
    for (int st = 0; st < 5; ++st) {
        const int o = 16 >> st, m = 16 >> st;   // partner distance, columns kept
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = up ? v[i] : v[i + m];
            const float keep = up ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0];
}

// Column sums of a 32-row x 16-column block held one row per lane (v[i] =
// column i): recursive halving keeps, at each step, the half of the columns
// selected by one lane bit and adds the partner's other half; after four
// steps lanes l and l ^ 1 hold partial sums of column l >> 1 over the lanes
// of their parity, and one more exchange completes both (16 shuffles).
__device__ __forceinline__ float column_sum16(float (&v)[16], int lane)
{
#pragma unroll
    for (int st = 0; st < 4; ++st) {
        const int o = 16 >> st, m = 8 >> st;   // partner distance, columns kept
        const bool up = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < m; ++i) {
            const float send = up ? v[i] : v[i + m];
            const float keep = up ? v[i + m] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 1);
}

// ---- state pass: shared memory (offsets from a 1024-byte aligned base)
constexpr uint32_t kSOffX = 0;             // X [row][p]      16 KB (TMA), then w o X in place
constexpr uint32_t kSOffB = 16384;         // B [row][n]      2 x 16 KB (TMA)
constexpr uint32_t kSOffS = 49152;         // S_in^T [n][p]   16 KB (to the workspace)
constexpr uint32_t kSOffVec = 65536;       // f32 c[128] (log2 units, by row), dt[128]
constexpr uint32_t kSOffMbar = kSOffVec + 1024;
constexpr uint32_t kSOffTmem = kSOffMbar + 16;
constexpr uint32_t kSSmem = kSOffTmem + 16 + 1024;

// The chunk's prefix sums of dt A (log2 units) by tile row, from one warp:
// lane l takes walk slots 4l .. 4l+3.  cumw (if given) gets the prefix sums
// of dt itself by walk slot.
__device__ __forceinline__ void chunk_prefix(const float *dtv, float *cv, float *cumw, float a2, bool rev,
                                             int lane)
{
    float v[4], run = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        run += dtv[rev ? kBQ - 1 - j : j];
        v[i] = run;
    }
    float incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    const float excl = incl - run;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int j = 4 * lane + i;
        cv[rev ? kBQ - 1 - j : j] = a2 * (excl + v[i]);
        if (cumw) cumw[j] = excl + v[i];
    }
}

}  // namespace

// The state entering every chunk of one (head, sequence, direction) walk,
// as bf16 S_in^T tiles.  S^T (lane n, 64 columns p) lives in tensor memory;
// per chunk: S_in^T -> tile, S^T <- e^{c_last} S^T + B^T (w o X).
__global__ void __launch_bounds__(kBThreads, 3)
bwd_tc_state_kernel(const __grid_constant__ CUtensorMap tm_act_f, const __grid_constant__ CUtensorMap tm_act_r,
                    const BwdTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & (kBQ - 1), hw = tid >> 7;
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    const bool rev = dir != 0;
    const int L = p.len, H = p.H;
    const CUtensorMap *tm = rev ? &tm_act_r : &tm_act_f;
    float *cv = reinterpret_cast<float *>(sm + kSOffVec);
    float *dtv = cv + kBQ;
    const uint32_t mb_in = sbase + kSOffMbar, mb_mma = mb_in + 8;
    const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    if (tid == 0) {
        tc::mbar_init(mb_in, 1);
        tc::mbar_init(mb_mma, 1);
        tc::prefetch_tmap(tm);
    }
    if (warp == 0) tc::tmem_alloc(sbase + kSOffTmem, 64);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kSOffTmem);
    const uint32_t my_cols = tmem + lane_base + 32 * hw;   // S^T[n = r][p = 32 hw ..]
    {
        // the state entering the walk: the caller's (forward) or zero
        const float *init = (!rev && p.init) ? p.init + ((size_t)b * H + h) * kBP * kBN : nullptr;
        uint32_t v[16];
#pragma unroll 1
        for (int g = 0; g < 2; ++g) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                v[i] = __float_as_uint(init ? init[(size_t)(32 * hw + 16 * g + i) * kBN + r] : 0.0f);
            tc::tmem_st16_nw(my_cols + 16 * g, v);
        }
        tc::tmem_wait_st();
    }
    const float a2 = p.A[h] * kLog2e;
    __nv_bfloat16 *tiles = p.states + (((size_t)dir * p.batch + b) * H + h) * p.nchunks * (kTileBytes / 2);
    bool ok = true;
#pragma unroll 1
    for (int k = 0; k < p.nchunks && ok; ++k) {
        const int t0 = rev ? L - kBQ * (k + 1) : kBQ * k;   // token of tile row 0
        if (tid == 0) {
            tc::mbar_expect_tx(mb_in, 3 * 16384);
            tc::tma_load_3d(sbase + kSOffX, tm, h * kBP, t0, b, mb_in);
            tc::tma_load_3d(sbase + kSOffB, tm, H * kBP, t0, b, mb_in);
            tc::tma_load_3d(sbase + kSOffB + 16384, tm, H * kBP + 64, t0, b, mb_in);
            if (k + 1 < p.nchunks) {
                const int tn = max(rev ? L - kBQ * (k + 2) : kBQ * (k + 1), 0);   // the next chunk, into L2
                tc::tma_prefetch_l2_3d(tm, h * kBP, tn, b);
                tc::tma_prefetch_l2_3d(tm, H * kBP, tn, b);
                tc::tma_prefetch_l2_3d(tm, H * kBP + 64, tn, b);
            }
        }
        if (tid < kBQ) {
            const int tok = t0 + r;
            dtv[r] = (tok >= 0 && tok < L) ? __bfloat162float(p.dt[((size_t)b * L + tok) * H + h]) : 0.0f;
        }
        __syncthreads();
        if (warp == 0) chunk_prefix(dtv, cv, nullptr, a2, rev, lane);
        if (tid == 0) ok = tc::mbar_wait_bounded(mb_in, k & 1, kBWait);
        ok = __syncthreads_and(ok);
        if (!ok) break;
        const float clast = cv[rev ? 0 : kBQ - 1];
        {
            // S_in^T row n = r (this half's 32 p) -> tile; S^T <- e^{c_last} S^T
            uint32_t sr[32];
            tc::tmem_ld32_nw(my_cols, sr);
            tc::tmem_wait_ld(sr);
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(sr[8 * pc + i]);
                *reinterpret_cast<uint4 *>(sm + kSOffS + tc::sw128(r, 4 * hw + pc)) = pack8(f);
            }
            const float al = tc::exp2_approx(clast);
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                uint32_t v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(sr[16 * g + i]) * al);
                tc::tmem_st16_nw(my_cols + 16 * g, v);
            }
            // row s = r of w o X (this half's 32 p)
            const float ws = tc::exp2_approx(fminf(clast - cv[r], 0.0f)) * dtv[r];
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                const uint32_t off = tc::sw128(r, 4 * hw + pc);
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + kSOffX + off), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] *= ws;
                *reinterpret_cast<uint4 *>(sm + kSOffX + off) = pack8(f);   // (this thread's half row only)
            }
            tc::tmem_wait_st();
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            tc::bulk_store(tiles + (size_t)k * (kTileBytes / 2), sbase + kSOffS, kTileBytes);
            tc::bulk_commit();
            // S^T[n][p] += sum_s B[s][n] (w o X)[s][p]: A = B read MN-major (M = n),
            // B operand = w o X MN-major (N = p)
            const uint64_t dBmn = tc::smem_desc(sbase + kSOffB, 16384, 1024);
            const uint64_t dWX = tc::smem_desc(sbase + kSOffX, 1024, 1024);
            constexpr uint32_t idS = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < kBQ / 16; ++ks)
                tc::mma_bf16(tmem, tc::desc_add(dBmn, ks * 2048), tc::desc_add(dWX, ks * 2048), idS, 1);
            tc::mma_commit(mb_mma);
            ok = tc::mbar_wait_bounded(mb_mma, k & 1, kBWait);
            tc::bulk_wait_read0();   // the tile is out of shared memory
        }
        ok = __syncthreads_and(ok);
        tc::fence_after_sync();
    }
    if (tid == 0) tc::bulk_wait0();
    if (!ok && tid == 0) record_error(p.status, kStatusTimeout);
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

namespace {

// ---- adjoint pass: shared memory
constexpr uint32_t kAOffX = 0;          // X [row][p] 16 KB (TMA); later w o X in place
constexpr uint32_t kAOffDY = 16384;     // dY [row][p] 16 KB (TMA); later e^c o dY in place
constexpr uint32_t kAOffB = 32768;      // B [row][n] 2 x 16 KB (TMA)
constexpr uint32_t kAOffC = 65536;      // C [row][n] 2 x 16 KB (TMA)
constexpr uint32_t kAOffW = 98304;      // W [t][s] 2 x 16 KB
constexpr uint32_t kAOffT = 131072;     // T [t][s] 2 x 16 KB
constexpr uint32_t kAOffSin = 163840;   // S_in^T [n][p] 16 KB (bulk copy)
constexpr uint32_t kAOffDS = 180224;    // dS^T [n][p] 16 KB (bf16 copy of the TMEM adjoint)
constexpr uint32_t kAOffVec = 196608;   // f32 vectors (below)
// f32 vectors (offsets in floats; see the kernel)
constexpr int kVCv = 0, kVDt = kVCv + kBQ, kVCum = kVDt + kBQ, kVRsp = kVCum + kBQ, kVDdp = kVRsp + 4 * kBQ,
              kVCsp = kVDdp + 4 * kBQ, kVXbp = kVCsp + 4 * kBQ, kVSdp = kVXbp + 4 * kBQ, kVDcw = kVSdp + 4 * kBQ,
              kVGdw = kVDcw + kBQ, kVUw = kVGdw + kBQ, kVRed = kVUw + kBQ;
constexpr int kVecFloats = kVRed + 64;
constexpr uint32_t kAOffMbar = kAOffVec + 4 * kVecFloats;
constexpr uint32_t kAOffTmem = kAOffMbar + 32;
constexpr uint32_t kASmem = kAOffTmem + 16 + 1024;
static_assert(kASmem <= 232448, "shared memory of the adjoint pass");

// tensor memory columns (512 allocated)
constexpr uint32_t kColCB = 0;      // C B^T (t, s); then dB (s, n)
constexpr uint32_t kColDYX = 128;   // dY X^T (t, s); then dC (t, n)
constexpr uint32_t kColCS = 256;    // C S_in^T (t, p)
constexpr uint32_t kColDX1 = 320;   // W^T dY (s, p)
constexpr uint32_t kColDX2 = 384;   // B dS^T (s, p)
constexpr uint32_t kColDS = 448;    // dS^T (n, p), fp32, carried across chunks

}  // namespace

// The chunked adjoint of one (head, sequence, direction) walk, from its last
// chunk.  Phases per chunk (thread 0 issues every MMA and TMA load):
//  P1  C B^T, dY X^T, C S_in^T, B dS^T
//  P2  W, T (bf16 tiles), row and column sums for dt, the per-row dot
//      products, w o X in place
//  P3  dX1 = W^T dY, dB = T^T C + (w o X) dS, dC = T B
//  P4  dX and dB out, dt and A, e^c o dY in place, dS^T <- e^{c_last} dS^T
//  P5  dC += (e^c o dY) S_in, dS^T += C^T (e^c o dY)
//  P6  dC out
__global__ void __launch_bounds__(kAThreads, 1)
bwd_tc_scan_kernel(const __grid_constant__ CUtensorMap tm_act_f, const __grid_constant__ CUtensorMap tm_act_r,
                   const __grid_constant__ CUtensorMap tm_dy, const __grid_constant__ CUtensorMap tm_dact_f,
                   const __grid_constant__ CUtensorMap tm_dact_r, const BwdTcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int r = tid & (kBQ - 1), qc = tid >> 7, quarter = warp & 3;
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    const bool rev = dir != 0;
    const int L = p.len, H = p.H, ch = p.ch, nc = p.nchunks;
    const CUtensorMap *tm = rev ? &tm_act_r : &tm_act_f;
    const CUtensorMap *tmd = rev ? &tm_dact_r : &tm_dact_f;   // fp32 gradient, for the B/C reductions
    float *dact = rev ? p.dact[1] : p.dact[0];
    float *vec = reinterpret_cast<float *>(sm + kAOffVec);
    float *cv = vec + kVCv;       // [128] c (log2 units) by row
    float *dtv = vec + kVDt;      // [128] dt by row
    float *cumw = vec + kVCum;    // [128] prefix sums of dt by walk slot
    float *rsp = vec + kVRsp;     // [4][128] row sums of dY X^T o W, per column quarter
    float *ddp = vec + kVDdp;     // [4][128] column sums of dY X^T o C B^T o e, per row quarter
    float *csp = vec + kVCsp;     // [4][128] dY_t . (C S_in^T)_t per quarter
    float *xbp = vec + kVXbp;     // [4][128] x_s . (B dS^T)_s per quarter
    float *sdp = vec + kVSdp;     // [4][128] <dS^T, S_in^T> of row n per quarter
    float *dcw = vec + kVDcw;     // [128] dL/dc by walk slot
    float *gdw = vec + kVGdw;     // [128] direct dt terms by walk slot
    float *uw = vec + kVUw;       // [128] U_s by row
    float *red = vec + kVRed;     // [64] reductions
    const uint32_t mb_in = sbase + kAOffMbar, mb_p1 = mb_in + 8, mb_p3 = mb_in + 16, mb_p5 = mb_in + 24;
    const uint32_t lane_base = static_cast<uint32_t>(32 * quarter) << 16;
    if (tid == 0) {
        tc::mbar_init(mb_in, 1);
        tc::mbar_init(mb_p1, 1);
        tc::mbar_init(mb_p3, 1);
        tc::mbar_init(mb_p5, 1);
        tc::prefetch_tmap(tm);
        tc::prefetch_tmap(&tm_dy);
        tc::prefetch_tmap(tmd);
    }
    if (warp == 0) tc::tmem_alloc(sbase + kAOffTmem, 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kAOffTmem);
    const uint32_t trow = tmem + lane_base;   // this thread's TMEM lane, column 0
    {
        // no adjoint flows into the state leaving the walk
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tc::tmem_st16_nw(trow + kColDS + 16 * qc, z);
        tc::tmem_wait_st();
    }
    const float a2 = p.A[h] * kLog2e, Aa = p.A[h], Dh = p.D[h];
    const __nv_bfloat16 *tiles = p.states + (((size_t)dir * p.batch + b) * H + h) * nc * (kTileBytes / 2);
    float dA_acc = 0.0f, dD_acc = 0.0f;
    bool ok = true;
#pragma unroll 1
    for (int k = nc - 1; k >= 0; --k) {
        const uint32_t par = (uint32_t)(nc - 1 - k) & 1u;   // mbarrier phase of this iteration
        const int t0 = rev ? L - kBQ * (k + 1) : kBQ * k;  // token of tile row 0
        const int tok = t0 + r;
        const bool tok_ok = tok >= 0 && tok < L;
        // ---- P0: this chunk's tiles, dt, and the bf16 copy of dS^T
        // staging rows of the fp32 dB / dC tiles: row q is token t0 + off + q
        // (the reverse walk's last chunk starts before token 0; a tensor
        // reduction may not start at a negative row, so its box starts at
        // token 0 and the rows past the chunk are zeros)
        const int off = t0 < 0 ? -t0 : 0;
        const int q = (r - off) & (kBQ - 1);
        if (tid == 0) {
            // dY and C first (no staging lives there), then X, B and S_in once
            // the last chunk's dB / dC staging in them has been read
            tc::mbar_expect_tx(mb_in, 7 * 16384);
            tc::tma_load_3d(sbase + kAOffDY, &tm_dy, h * kBP, t0, b, mb_in);
            tc::tma_load_3d(sbase + kAOffC, tm, H * kBP + kBN, t0, b, mb_in);
            tc::tma_load_3d(sbase + kAOffC + 16384, tm, H * kBP + kBN + 64, t0, b, mb_in);
            tc::bulk_wait_read0();
            tc::tma_load_3d(sbase + kAOffX, tm, h * kBP, t0, b, mb_in);
            tc::tma_load_3d(sbase + kAOffB, tm, H * kBP, t0, b, mb_in);
            tc::tma_load_3d(sbase + kAOffB + 16384, tm, H * kBP + 64, t0, b, mb_in);
            tc::bulk_load(sbase + kAOffSin, tiles + (size_t)k * (kTileBytes / 2), kTileBytes, mb_in);
            if (k > 0) {
                // the next chunk's tiles into L2 (its loads are issued only once
                // this chunk is done with the buffers)
                const int tn = rev ? L - kBQ * k : kBQ * (k - 1);
                tc::tma_prefetch_l2_3d(tm, h * kBP, tn, b);
                tc::tma_prefetch_l2_3d(&tm_dy, h * kBP, tn, b);
#pragma unroll
                for (int j = 0; j < 4; ++j) tc::tma_prefetch_l2_3d(tm, H * kBP + 64 * j, tn, b);
                tc::bulk_prefetch_l2(tiles + (size_t)(k - 1) * (kTileBytes / 2), kTileBytes);
            }
        }
        if (tid < kBQ) dtv[r] = tok_ok ? __bfloat162float(p.dt[((size_t)b * L + tok) * H + h]) : 0.0f;
        {
            uint32_t v[16];
            tc::tmem_ld16_nw(trow + kColDS + 16 * qc, v);
            tc::tmem_wait_ld16(v);
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                float f[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(v[8 * pc + i]);
                *reinterpret_cast<uint4 *>(sm + kAOffDS + tc::sw128(r, 2 * qc + pc)) = pack8(f);
            }
        }
        tc::fence_proxy_async();
        __syncthreads();
        if (warp == 0) chunk_prefix(dtv, cv, cumw, a2, rev, lane);
        // ---- P1
        if (tid == 0) {
            ok = tc::mbar_wait_bounded(mb_in, par, kBWait);
            if (ok) {
                tc::fence_after_sync();
                const uint64_t dCk = tc::smem_desc(sbase + kAOffC, 16, 1024);
                const uint64_t dBk = tc::smem_desc(sbase + kAOffB, 16, 1024);
                const uint64_t dYk = tc::smem_desc(sbase + kAOffDY, 16, 1024);
                const uint64_t dXk = tc::smem_desc(sbase + kAOffX, 16, 1024);
                const uint64_t dSinMN = tc::smem_desc(sbase + kAOffSin, 1024, 1024);
                const uint64_t dDSMN = tc::smem_desc(sbase + kAOffDS, 1024, 1024);
                constexpr uint32_t idQQ = tc::idesc_bf16(128, 128, 0, 0);
                constexpr uint32_t idQP = tc::idesc_bf16(128, 64, 0, 1);
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    tc::mma_bf16(tmem + kColCB, tc::desc_add(dCk, koff), tc::desc_add(dBk, koff), idQQ, ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < kBP / 16; ++ks)
                    tc::mma_bf16(tmem + kColDYX, tc::desc_add(dYk, ks * 32), tc::desc_add(dXk, ks * 32), idQQ,
                                 ks > 0);
#pragma unroll
                for (int ks = 0; ks < kBN / 16; ++ks) {
                    const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                    tc::mma_bf16(tmem + kColCS, tc::desc_add(dCk, koff), tc::desc_add(dSinMN, ks * 2048), idQP,
                                 ks > 0);
                    tc::mma_bf16(tmem + kColDX2, tc::desc_add(dBk, koff), tc::desc_add(dDSMN, ks * 2048), idQP,
                                 ks > 0);
                }
                tc::mma_commit(mb_p1);
                ok = tc::mbar_wait_bounded(mb_p1, par, kBWait);
            }
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        const float ct = cv[r];
        const float clast = cv[rev ? 0 : kBQ - 1];
        // ---- P2: W and T of row t = r, columns s = 32 qc .. 32 qc + 31 (two
        // passes of 16)
        {
            float rs = 0.0f;
#pragma unroll 1
            for (int g = 0; g < 2; ++g) {
                const int s0 = 32 * qc + 16 * g;
                uint32_t cb[16], yx[16];
                tc::tmem_ld16_nw(trow + kColCB + s0, cb);
                tc::tmem_ld16_nw(trow + kColDYX + s0, yx);
                tc::tmem_wait_ld16(cb);
                tc::tmem_wait_ld16(yx);
                // pd = dY X^T o C B^T o e; its row sums weighted by dt_s (rs) and
                // its column sums (times dt_s: those of dY X^T o W) feed dL/dc
                float pd[16];
                uint32_t wp[8], tp[8];
#pragma unroll
                for (int i4 = 0; i4 < 4; ++i4) {
                    const float4 c4 = *reinterpret_cast<const float4 *>(cv + s0 + 4 * i4);
                    const float4 d4 = *reinterpret_cast<const float4 *>(dtv + s0 + 4 * i4);
                    const float cs_[4] = {c4.x, c4.y, c4.z, c4.w};
                    const float ds_[4] = {d4.x, d4.y, d4.z, d4.w};
                    float wv[4], tv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int i = 4 * i4 + e, s = s0 + i;
                        const bool in = rev ? (s >= r) : (s <= r);   // walk slot of s <= that of t
                        const float dec = in ? tc::exp2_approx(fminf(ct - cs_[e], 0.0f)) : 0.0f;
                        const float cbe = __uint_as_float(cb[i]) * dec;
                        const float yxv = __uint_as_float(yx[i]);
                        wv[e] = cbe * ds_[e];
                        tv[e] = yxv * dec * ds_[e];
                        pd[i] = yxv * cbe;
                        rs = fmaf(pd[i], ds_[e], rs);
                    }
                    wp[2 * i4] = tc::pack_bf16x2(wv[0], wv[1]);
                    wp[2 * i4 + 1] = tc::pack_bf16x2(wv[2], wv[3]);
                    tp[2 * i4] = tc::pack_bf16x2(tv[0], tv[1]);
                    tp[2 * i4 + 1] = tc::pack_bf16x2(tv[2], tv[3]);
                }
                // columns s0 .. s0+15: 64-column panel qc >> 1, 8-column pieces
                // 4 (qc & 1) + 2 g + pc
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    const uint32_t off = (qc >> 1) * 16384 + tc::sw128(r, 4 * (qc & 1) + 2 * g + pc);
                    *reinterpret_cast<uint4 *>(sm + kAOffW + off) =
                        make_uint4(wp[4 * pc], wp[4 * pc + 1], wp[4 * pc + 2], wp[4 * pc + 3]);
                    *reinterpret_cast<uint4 *>(sm + kAOffT + off) =
                        make_uint4(tp[4 * pc], tp[4 * pc + 1], tp[4 * pc + 2], tp[4 * pc + 3]);
                }
                const float csum = column_sum16(pd, lane);
                if ((lane & 1) == 0) ddp[quarter * kBQ + s0 + (lane >> 1)] = csum;
            }
            rsp[qc * kBQ + r] = rs;
        }
        // per-row dot products over this quarter's 16 p: dY_t . (C S_in^T)_t,
        // x_s . (B dS^T)_s, dY . x (for D), and <dS^T, S_in^T> of row n = r
        {
            uint32_t cs[16], x2[16], ds[16];
            tc::tmem_ld16_nw(trow + kColCS + 16 * qc, cs);
            tc::tmem_ld16_nw(trow + kColDX2 + 16 * qc, x2);
            tc::tmem_ld16_nw(trow + kColDS + 16 * qc, ds);
            tc::tmem_wait_ld16(cs);
            tc::tmem_wait_ld16(x2);
            tc::tmem_wait_ld16(ds);
            float a_cs = 0.0f, a_xb = 0.0f, a_dd = 0.0f, a_sd = 0.0f;
            const float ws = tc::exp2_approx(fminf(clast - ct, 0.0f)) * dtv[r];
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                const uint32_t off = tc::sw128(r, 2 * qc + pc);
                float yv[8], xv[8], sv[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + kAOffDY + off), yv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + kAOffX + off), xv);
                unpack8(*reinterpret_cast<const uint4 *>(sm + kAOffSin + off), sv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    a_cs = fmaf(yv[i], __uint_as_float(cs[8 * pc + i]), a_cs);
                    a_xb = fmaf(xv[i], __uint_as_float(x2[8 * pc + i]), a_xb);
                    a_dd = fmaf(yv[i], xv[i], a_dd);
                    a_sd = fmaf(__uint_as_float(ds[8 * pc + i]), sv[i], a_sd);
                    xv[i] *= ws;
                }
                // w o X in place (this thread is the last reader of its quarter row)
                *reinterpret_cast<uint4 *>(sm + kAOffX + off) = pack8(xv);
            }
            csp[qc * kBQ + r] = a_cs;
            xbp[qc * kBQ + r] = a_xb;
            sdp[qc * kBQ + r] = a_sd;
            dD_acc += a_dd;
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        // ---- P3
        if (tid == 0) {
            tc::fence_after_sync();
            const uint64_t dWmn = tc::smem_desc(sbase + kAOffW, 16384, 1024);
            const uint64_t dTmn = tc::smem_desc(sbase + kAOffT, 16384, 1024);
            const uint64_t dTk = tc::smem_desc(sbase + kAOffT, 16, 1024);
            const uint64_t dYmn = tc::smem_desc(sbase + kAOffDY, 1024, 1024);
            const uint64_t dCmn = tc::smem_desc(sbase + kAOffC, 16384, 1024);
            const uint64_t dBmn = tc::smem_desc(sbase + kAOffB, 16384, 1024);
            const uint64_t dXk = tc::smem_desc(sbase + kAOffX, 16, 1024);
            const uint64_t dDSk = tc::smem_desc(sbase + kAOffDS, 16, 1024);
            constexpr uint32_t idX1 = tc::idesc_bf16(128, 64, 1, 1);
            constexpr uint32_t idTC = tc::idesc_bf16(128, 128, 1, 1);
            constexpr uint32_t idQQ = tc::idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idTB = tc::idesc_bf16(128, 128, 0, 1);
#pragma unroll
            for (int ks = 0; ks < kBQ / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kColDX1, tc::desc_add(dWmn, ks * 2048), tc::desc_add(dYmn, ks * 2048), idX1,
                             ks > 0);
                tc::mma_bf16(tmem + kColCB, tc::desc_add(dTmn, ks * 2048), tc::desc_add(dCmn, ks * 2048), idTC,
                             ks > 0);
                tc::mma_bf16(tmem + kColDYX, tc::desc_add(dTk, koff), tc::desc_add(dBmn, ks * 2048), idTB, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < kBP / 16; ++ks)
                tc::mma_bf16(tmem + kColCB, tc::desc_add(dXk, ks * 32), tc::desc_add(dDSk, ks * 32), idQQ, 1);
            tc::mma_commit(mb_p3);
            ok = tc::mbar_wait_bounded(mb_p3, par, kBWait);
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        // ---- P4: dX of row s = r (this quarter's 16 p), dB of row s (32 n)
        const float ws = tc::exp2_approx(fminf(clast - ct, 0.0f)) * dtv[r];
        {
            uint32_t a1[16], a2v[16];
            tc::tmem_ld16_nw(trow + kColDX1 + 16 * qc, a1);
            tc::tmem_ld16_nw(trow + kColDX2 + 16 * qc, a2v);
            tc::tmem_wait_ld16(a1);
            tc::tmem_wait_ld16(a2v);
            const float ec = tc::exp2_approx(fminf(ct, 0.0f));
            float4 *dst = reinterpret_cast<float4 *>(dact + ((size_t)b * L + tok) * ch + h * kBP + 16 * qc);
            // the rows leave by two TMA stores of 32-column fp32 boxes (128-byte
            // swizzle) staged in the X and dS tiles, which the products have
            // finished with; a chunk whose first row lies before token 0 (the
            // reverse walk's short chunk: a store may not start at a negative
            // row) by per-thread stores
            uint8_t *xbox = sm + ((qc >> 1) ? kAOffDS : kAOffX);
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                const uint32_t soff = tc::sw128(r, 2 * qc + pc);
                float yv[8], o[8];
                unpack8(*reinterpret_cast<const uint4 *>(sm + kAOffDY + soff), yv);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int q = 8 * pc + i;
                    o[i] = __uint_as_float(a1[q]) + Dh * yv[i] + ws * __uint_as_float(a2v[q]);
                    yv[i] *= ec;
                }
                if (off == 0) {
                    const int c0 = 4 * (qc & 1) + 2 * pc;
                    *reinterpret_cast<float4 *>(xbox + tc::sw128(r, c0)) = make_float4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<float4 *>(xbox + tc::sw128(r, c0 + 1)) = make_float4(o[4], o[5], o[6], o[7]);
                } else if (tok_ok) {
                    dst[2 * pc] = make_float4(o[0], o[1], o[2], o[3]);
                    dst[2 * pc + 1] = make_float4(o[4], o[5], o[6], o[7]);
                }
                // e^c o dY in place (this thread is the last reader of its quarter row)
                *reinterpret_cast<uint4 *>(sm + kAOffDY + soff) = pack8(yv);
            }
        }
        // dB rows staged as four 32-column fp32 boxes (128-byte swizzle) in the
        // W and T tiles, which the products above have finished with
        {
            // box qc: columns 32 qc .. 32 qc + 31
            uint32_t v[32];
            tc::tmem_ld32_nw(trow + kColCB + 32 * qc, v);
            tc::tmem_wait_ld(v);
            uint8_t *box = sm + (qc < 2 ? kAOffW : kAOffT) + 16384 * (qc & 1);
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(box + tc::sw128(q, c)) =
                    r >= off ? make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]) : make_uint4(0u, 0u, 0u, 0u);
        }
        {
            // dS^T <- e^{c_last} dS^T (its bf16 copy was taken in P0)
            uint32_t v[16];
            tc::tmem_ld16_nw(trow + kColDS + 16 * qc, v);
            tc::tmem_wait_ld16(v);
            const float al = tc::exp2_approx(clast);
            uint32_t u[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(__uint_as_float(v[i]) * al);
            tc::tmem_st16_nw(trow + kColDS + 16 * qc, u);
        }
        if (qc == 0) {
            // dL/dc and the direct dt terms of row r, by walk slot
            const int j = rev ? kBQ - 1 - r : r;
            const float xb = (xbp[r] + xbp[kBQ + r]) + (xbp[2 * kBQ + r] + xbp[3 * kBQ + r]);
            const float el = tc::exp2_approx(fminf(clast - ct, 0.0f));
            const float u = el * dtv[r] * xb;
            const float dsum = ddp[r] + ddp[kBQ + r] + ddp[2 * kBQ + r] + ddp[3 * kBQ + r];
            const float csum = dsum * dtv[r];   // column sum of dY X^T o W
            const float cs4 = (csp[r] + csp[kBQ + r]) + (csp[2 * kBQ + r] + csp[3 * kBQ + r]);
            const float rs4 = (rsp[r] + rsp[kBQ + r]) + (rsp[2 * kBQ + r] + rsp[3 * kBQ + r]);
            dcw[j] = tc::exp2_approx(fminf(ct, 0.0f)) * cs4 - u + rs4 - csum;
            gdw[j] = dsum + el * xb;
            uw[r] = u;
        }
        tc::fence_proxy_async();
        tc::tmem_wait_st();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            if (off == 0) {
                // dX of this head's x columns (written: no other pass adds to them)
                tc::tma_store_3d(tmd, sbase + kAOffX, h * kBP, t0, b);
                tc::tma_store_3d(tmd, sbase + kAOffDS, h * kBP + 32, t0, b);
                tc::bulk_commit();
            }
            // dB += this head's rows (fp32 reductions at L2)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                tc::tma_reduce_add_3d(tmd, sbase + (j < 2 ? kAOffW : kAOffT) + 16384 * (j & 1), H * kBP + 32 * j,
                                      t0 + off, b);
            tc::bulk_commit();
        }
        if (warp == 0) {
            // the chunk's last walk slot also carries e^{c_last} <dS, S_in> + sum_s U_s;
            // then dt gets A times the suffix sums of dL/dc (walk order), A the
            // sum of dL/dc_j times the prefix sums of dt
            float sd = 0.0f, us = 0.0f;
#pragma unroll
            for (int i = lane; i < kBQ; i += 32) {
                sd += (sdp[i] + sdp[kBQ + i]) + (sdp[2 * kBQ + i] + sdp[3 * kBQ + i]);
                us += uw[i];
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                sd += __shfl_xor_sync(0xffffffffu, sd, o);
                us += __shfl_xor_sync(0xffffffffu, us, o);
            }
            float d[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) d[i] = dcw[4 * lane + i];
            if (lane == 31) d[3] += tc::exp2_approx(clast) * sd + us;
            float suf[4], run = 0.0f;
#pragma unroll
            for (int i = 3; i >= 0; --i) {
                run += d[i];
                suf[i] = run;
            }
            float incl = run;   // suffix over lanes >= this one
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_down_sync(0xffffffffu, incl, o);
                if (lane + o < 32) incl += v;
            }
            const float after = incl - run;   // lanes above this one
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j = 4 * lane + i;
                const int wk = kBQ * k + j;   // walk index
                if (wk < L) {
                    const int tk = rev ? L - 1 - wk : wk;
                    atomicAdd(p.ddt + ((size_t)b * L + tk) * H + h, gdw[j] + Aa * (suf[i] + after));
                }
                dA_acc = fmaf(d[i], cumw[j], dA_acc);
            }
        }
        // ---- P5
        if (tid == 0) {
            tc::fence_after_sync();
            const uint64_t dYk = tc::smem_desc(sbase + kAOffDY, 16, 1024);
            const uint64_t dSink = tc::smem_desc(sbase + kAOffSin, 16, 1024);
            const uint64_t dCmn = tc::smem_desc(sbase + kAOffC, 16384, 1024);
            const uint64_t dYmn = tc::smem_desc(sbase + kAOffDY, 1024, 1024);
            constexpr uint32_t idQQ = tc::idesc_bf16(128, 128, 0, 0);
            constexpr uint32_t idS = tc::idesc_bf16(128, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < kBP / 16; ++ks)
                tc::mma_bf16(tmem + kColDYX, tc::desc_add(dYk, ks * 32), tc::desc_add(dSink, ks * 32), idQQ, 1);
#pragma unroll
            for (int ks = 0; ks < kBQ / 16; ++ks)
                tc::mma_bf16(tmem + kColDS, tc::desc_add(dCmn, ks * 2048), tc::desc_add(dYmn, ks * 2048), idS, 1);
            tc::mma_commit(mb_p5);
            ok = tc::mbar_wait_bounded(mb_p5, par, kBWait);
            tc::bulk_wait_read1();   // the dX stores have read the X tile (dC is staged there)
        }
        ok = __syncthreads_and(ok);
        if (!ok) break;
        tc::fence_after_sync();
        // ---- P6: dC of row t = r (64 n), staged like dB in the X, B and S_in
        // tiles (every product that reads them is done; the next chunk's
        // loads into them wait for the reductions to read them)
        {
            uint32_t v[32];
            tc::tmem_ld32_nw(trow + kColDYX + 32 * qc, v);
            tc::tmem_wait_ld(v);
            const int j = qc;   // box j: columns 32 j .. 32 j + 31
            uint8_t *box = sm + (j == 0 ? kAOffX : j == 3 ? kAOffSin : kAOffB + 16384 * (j - 1));
#pragma unroll
            for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4 *>(box + tc::sw128(q, c)) =
                    r >= off ? make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]) : make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async();
        tc::fence_before_sync();
        __syncthreads();
        if (tid == 0) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                tc::tma_reduce_add_3d(tmd, sbase + (j == 0 ? kAOffX : j == 3 ? kAOffSin : kAOffB + 16384 * (j - 1)),
                                      H * kBP + kBN + 32 * j, t0 + off, b);
            tc::bulk_commit();
        }
    }
    if (tid == 0) tc::bulk_wait0();   // every reduction written
    if (ok) {
        if (!rev && p.dinit) {
            // the adjoint of the caller's initial state: dinit[p][n] = dS^T[n][p]
            uint32_t v[16];
            tc::tmem_ld16_nw(trow + kColDS + 16 * qc, v);
            tc::tmem_wait_ld16(v);
            float *dst = p.dinit + ((size_t)b * H + h) * kBP * kBN;
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[(size_t)(16 * qc + i) * kBN + r] = __uint_as_float(v[i]);
        }
        // D and A of this head
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) dD_acc += __shfl_xor_sync(0xffffffffu, dD_acc, o);
        if (lane == 0) red[warp] = dD_acc;
        __syncthreads();
        if (tid == 0) {
            float s = 0.0f;
            for (int i = 0; i < kAThreads / 32; ++i) s += red[i];
            atomicAdd(p.dD + h, s);
        }
        if (warp == 0) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) dA_acc += __shfl_xor_sync(0xffffffffu, dA_acc, o);
            if (lane == 0) atomicAdd(p.dA + h, dA_acc);
        }
    } else if (tid == 0) {
        record_error(p.status, kStatusTimeout);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 512);
}

namespace {

PFN_cuTensorMapEncodeTiled_v12000 bwd_encode_fn()
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

// (batch, len, cols) bf16 or fp32, boxes of 128 bytes x 128 rows, 128-byte swizzle
bool make_tile_map(CUtensorMap *m, const void *base, uint64_t cols, uint64_t len, uint64_t batch,
                   bool f32 = false)
{
    auto fn = bwd_encode_fn();
    if (!fn) return false;
    const uint64_t esz = f32 ? 4 : 2;
    const cuuint64_t dims[3] = {cols, len, batch};
    const cuuint64_t strides[2] = {cols * esz, cols * len * esz};
    const cuuint32_t box[3] = {(cuuint32_t)(128 / esz), (cuuint32_t)kBQ, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
              const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool backward_tc_supported(const bimamba_dims &d)
{
    return d.dtype == BIMAMBA_BF16 && d.headdim == kBP && d.d_state == kBN && d.ngroups == 1 && d.d_conv == 4;
}

size_t backward_tc_state_bytes(const bimamba_dims &d)
{
    const size_t nchunks = ((size_t)d.len + kBQ - 1) / kBQ;
    return 2 * (size_t)d.batch * d.heads * nchunks * kTileBytes;
}

cudaError_t launch_backward_tc(const BackwardTcProblem &q, cudaStream_t s)
{
    const bimamba_dims &d = q.dims;
    BwdTcParams p;
    p.dt = static_cast<const __nv_bfloat16 *>(q.dt);
    p.A = q.A;
    p.D = q.D;
    p.init = q.init;
    p.states = static_cast<__nv_bfloat16 *>(q.states);
    p.dact[0] = q.dact[0];
    p.dact[1] = q.dact[1];
    p.ddt = q.ddt;
    p.dA = q.dA;
    p.dD = q.dD;
    p.dinit = q.dinit;
    p.status = device_status_word();
    p.batch = d.batch;
    p.len = d.len;
    p.H = d.heads;
    p.ch = d.heads * kBP + 2 * kBN;
    p.nchunks = (d.len + kBQ - 1) / kBQ;
    CUtensorMap tm_f, tm_r, tm_dy, tm_df, tm_dr;
    if (!make_tile_map(&tm_f, q.act[0], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch) ||
        !make_tile_map(&tm_r, q.act[1], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch) ||
        !make_tile_map(&tm_dy, q.dy, (uint64_t)d.heads * kBP, (uint64_t)d.len, (uint64_t)d.batch) ||
        !make_tile_map(&tm_df, q.dact[0], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, true) ||
        !make_tile_map(&tm_dr, q.dact[1], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, true))
        return cudaErrorInvalidValue;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(bwd_tc_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kSSmem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(bwd_tc_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kASmem)) != cudaSuccess)
        return e;
    const dim3 grid(d.heads, d.batch, 2);
    bwd_tc_state_kernel<<<grid, kBThreads, kSSmem, s>>>(tm_f, tm_r, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    const TimingEvents ev = timing_events();
    if (ev.start && (e = cudaEventRecord(ev.start, s)) != cudaSuccess) return e;
    bwd_tc_scan_kernel<<<grid, kAThreads, kASmem, s>>>(tm_f, tm_r, tm_dy, tm_df, tm_dr, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    if (ev.stop && (e = cudaEventRecord(ev.stop, s)) != cudaSuccess) return e;
    return cudaSuccess;
}

}  // namespace bimamba
