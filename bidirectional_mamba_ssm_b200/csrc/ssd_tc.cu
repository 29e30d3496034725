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
//     M[t,s] = G[t,s] exp(c_t - c_s) dt_s  (s < t),  G[t,t] dt_t + D  (s = t)
//     Y      = M X + diag(exp(c)) C S_in^T            (Q x P)
//     S_out  = exp(c_last) S_in + sum_s exp(c_last - c_s) dt_s x_s B_s^T
// The reverse stream is the same computation in walk order: chunk slots map
// to tokens through t = len-1-s; no flipped copy of any tensor is made.
//
// Mapping: one CTA owns (batch b, head pair, direction) and walks the chunks
// of its sequence (or of one segment of it).  Warps: 16 compute warps (512
// threads: conv, M, state scaling, epilogue), one producer warp (every MMA
// and TMA load, and the handshake releases) and one helper warp (dt copies,
// prefix sums and per-slot decay factors, up to two chunks ahead).  The two
// heads share B, C and G, so G is computed once per chunk for both.  Per
// chunk (all M = 128):
//     G        = C . B^T           A = C [t][n] K-major (smem), B = B [s][n] K-major
//     Yd_h     = M_h . X_h         A = M_h in TMEM,            B = X_h [s][p] MN-major
//     Yo       = C . [S_0;S_1]^T   A = C,                      B = S^T [n][p'] MN-major
//     S^T     += B^T . [wX_0|wX_1] A = B [s][n] MN-major,      B = wX [s][p'] MN-major
// The fp32 state S^T (n x p', both heads) lives in tensor memory: before the
// chunk's MMAs the threads scale it by exp(c_last) in place (and keep a bf16
// copy in shared memory as the Yo operand); the last MMA accumulates onto it.
// TMEM columns: G 0..127 (then Yd_0 0..63, Yd_1 64..127), M_0 128..191,
// M_1 192..255, Yo 256..383, S^T 384..511.
// Descriptors: K-major operands use stride 1024 B between 8-row groups; an
// MN-major operand uses leading offset = distance between its 64-element
// blocks along M/N (16 KB for the 128-wide tiles; for 64-wide tiles, which
// have a single block, the unused field is set equal to the 1024 B stride)
// and stride offset = 1024 B between groups of 8 rows along K.
// Decay factors: for s in a 32-slot block below t's block,
// exp(c_t - c_s) = exp(c_t - c_R) exp(c_R - c_s) with R the block's last
// slot; both factors are <= 1, so nothing overflows.  The diagonal 32 x 32
// blocks factorise the same way through 4-slot sub-blocks when the block's
// whole decay is at most 2^60 (so the row factor, >= 1 inside t's own
// sub-block, stays finite), else take one exponential per element.
//
// Forward+reverse sum: the two CTAs of a (b, head pair) meet per token chunk
// through a two-counter handshake in the caller's workspace: the first to
// finish a chunk writes its output (bf16), the second adds its own to it
// with bf16 reductions at L2.  The second one's wait is bounded; the first
// never waits.  (Untied directions with concatenated outputs, kConcat, do
// not meet: each direction stores its own half of every output row.)
#include "common.cuh"
#include "dispatch.h"
#include "tc_ptx.cuh"

#include <algorithm>
#include <cuda.h>
#include <cudaTypedefs.h>

namespace bimamba {

namespace {

constexpr int kQ = 128;       // chunk length
constexpr int kP = 64;        // headdim of this kernel
constexpr int kN = 128;       // d_state of this kernel
constexpr int kHeads = 2;     // heads per CTA
constexpr int kPP = kHeads * kP;   // x channels per CTA (128)
constexpr int kAluThreads = 512;          // compute group (16 warps)
constexpr int kProducerWarp = 16;         // issues every MMA and TMA load
constexpr int kProducerTid = 32 * kProducerWarp;
constexpr int kHelperWarp = 17;           // dt copies, prefix sums, slot factors
constexpr int kThreads = kAluThreads + 64;
constexpr int kBC = 2 * kN;   // B and C channels
constexpr int kRawRows = kQ + 3;   // raw x rows per chunk: 128 slots + 3-token conv halo
constexpr uint32_t kTmemCols = 512;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffC = 0;          // C      [t][n]   2 x 16 KB (TMA, swizzled)
constexpr uint32_t kOffB = 32768;      // B      [s][n]   2 x 16 KB (TMA, swizzled)
constexpr uint32_t kXbufBytes = 33792; // raw x [131][128] (TMA) -> X [s][p], 16 KB per head
constexpr uint32_t kOffXbuf0 = 65536;  // x buffer of even walk chunks
constexpr uint32_t kOffXbuf1 = kOffXbuf0 + kXbufBytes;   // odd walk chunks
constexpr uint32_t kOffXw = kOffXbuf1 + kXbufBytes;      // wX [s][p'] 2 x 16 KB
constexpr uint32_t kOffS = kOffXw + 32768;               // S^T bf16 [n][p'] 2 x 16 KB
constexpr uint32_t kRawBytes = kRawRows * kPP * 2;       // 33536
constexpr uint32_t kOffCum = kOffS + 32768;      // f32[2][2][128] prefix sums of dt*A (chunk parity, head)
constexpr uint32_t kOffDt = kOffCum + 2048;      // f32[2][2][128] dt
constexpr uint32_t kOffFB = kOffDt + 2048;       // f32[2][2][128] exp(c_R - c_s) dt_s, R = block end
constexpr uint32_t kOffWgt = kOffFB + 2048;      // f32[2][2][128] exp(c_last - c_s) dt_s
constexpr uint32_t kOffF4 = kOffWgt + 2048;      // f32[2][2][128] exp(c_R4 - c_s) dt_s, R4 = s | 3
constexpr uint32_t kOffConvW = kOffF4 + 2048;    // float4[128] conv taps of x
constexpr uint32_t kOffConvB = kOffConvW + 16 * kPP;   // f32[128]
constexpr uint32_t kOffMbar = kOffConvB + 4 * kPP;     // u64 x12 + 2 flag pointers (see the kernel)
constexpr uint32_t kOffTmem = kOffMbar + 112;    // u32 TMEM base
constexpr uint32_t kOffFlag = kOffTmem + 4;      // i32 handshake result
constexpr uint32_t kOffDtBuf = kOffFlag + 12;    // [2][128] bf16x2: dt of both heads, by cp.async
constexpr uint32_t kSmemUsed = kOffDtBuf + 2 * kQ * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;   // + alignment slack
constexpr uint32_t kBCBytes = 4 * kQ * 64 * 2;      // four 128 x 64 bf16 boxes
static_assert(kOffXbuf1 % 1024 == 0 && kOffXw % 1024 == 0 && kOffS % 1024 == 0, "tile alignment");
static_assert(kRawBytes <= kXbufBytes, "raw x tile must fit its buffer");

// TMEM columns: 0..255 hold G/Yd of one chunk and M of the other (the two
// 128-column regions alternate per chunk); Yo and the state are fixed.
constexpr uint32_t kColYo = 256;   // + 64 * head
constexpr uint32_t kColS = 384;    // + 64 * head

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz
constexpr int kArriveTid = 480;   // a thread outside warp 0 (which issues the MMAs)

// Per-direction inputs are indexed [0] forward stream, [1] reverse stream
// (the same pointers when the directions share their parameters); a CTA
// picks its direction's with a select, never a run-time array index.
struct TcParams {
    const __nv_bfloat16 *dt[2];
    const float *A[2];
    const float *D[2];
    const float *conv_w[2];
    const float *conv_b[2];
    const __nv_bfloat16 *tail;   // (batch, 4, ch) raw tokens before the sequence, or null
    const __nv_bfloat16 *head;   // (batch, 4, ch) raw tokens after it (sequence shards), or null
    const float *init;
    float *fin;
    __nv_bfloat16 *y;
    // sequence shards: every rank's shard end states from zero
    // [nranks][2 dir][batch][H][kP][kN] and log2 decays [nranks][2][batch][H]
    const float *shard_states;
    const float *shard_dec;
    int rank, nranks;
    int *flags;   // [batch][H/2][nchunks][2]: arrivals, partial-ready
    int *status;
    // segments (blockIdx.z): walk chunks [z * seg_chunks, +seg_chunks)
    float *seg_state;   // [dir][batch][H/2][nitems][2][kP][kN] item end states from zero
    float *seg_dec;     // [dir][batch][H/2][nitems][2] item decays, log2 units
    int seg_chunks;     // walk chunks per CTA
    int item_chunks;    // walk chunks per state-only item (0: no items)
    int nitems;
    int len, H, ch, nchunks, batch;
};

__device__ __forceinline__ int ld_acquire(const int *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Release store at GPU scope.  Issued by one thread after a CTA barrier, it
// publishes every write the CTA made before that barrier.
__device__ __forceinline__ void st_release(int *p, int v)
{
    asm volatile("st.release.gpu.global.b32 [%0], %1;" :: "l"(p), "r"(v) : "memory");
}

// Barrier over the compute group only (named barrier 1, 512 threads); the
// producer warp never joins it.
__device__ __forceinline__ void alu_sync()
{
    asm volatile("bar.sync 1, 512;" ::: "memory");
}

__device__ __forceinline__ bool alu_sync_and(bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %1, 0;\n\t"
        "bar.red.and.pred q, 1, 512, p;\n\t"
        "selp.b32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"((uint32_t)pred) : "memory");
    return r != 0;
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

// Prepass: conv+SiLU of the B and C channels, once per (sequence, direction),
// written in walk order: act[(dir * batch + b) * len + s][n], s = walk step
// (token s forward, token len-1-s reverse).  Without conv weights the raw
// values are copied.  One thread: 8 channels x 8 walk steps, 3-step window in
// registers; a warp covers one token's 256 channels (512 contiguous bytes).
__global__ void __launch_bounds__(128)
bc_prepass_kernel(const __nv_bfloat16 *__restrict__ xbc_f, const __nv_bfloat16 *__restrict__ xbc_r,
                  const __nv_bfloat16 *__restrict__ tail, const __nv_bfloat16 *__restrict__ head,
                  const float *__restrict__ conv_w_f,
                  const float *__restrict__ conv_w_r, const float *__restrict__ conv_b_f,
                  const float *__restrict__ conv_b_r, __nv_bfloat16 *__restrict__ act, int len,
                  int ch, int cbase, int batch)
{
    const int g = threadIdx.x & 31, sub = threadIdx.x >> 5;
    const int b = blockIdx.y;
    const bool rev = blockIdx.z != 0;
    // each direction's own raw input and conv parameters
    const __nv_bfloat16 *xbc = rev ? xbc_r : xbc_f;
    const float *conv_w = rev ? conv_w_r : conv_w_f;
    const float *conv_b = rev ? conv_b_r : conv_b_f;
    const int s_begin = blockIdx.x * 32 + sub * 8;
    if (s_begin >= len) return;
    const int s_end = min(s_begin + 8, len);
    const int n0 = 8 * g;
    const int c = cbase + n0;
    const __nv_bfloat16 *xb = xbc + (size_t)b * len * ch + c;
    __nv_bfloat16 *ob = act + ((size_t)(blockIdx.z * batch + b) * len) * kBC + n0;
    auto raw = [&](int s, float (&v)[8]) {
        if (s >= 0) {
            const int tok = rev ? len - 1 - s : s;
            unpack8(*reinterpret_cast<const uint4 *>(xb + (size_t)tok * ch), v);
        } else if (!rev && tail) {
            unpack8(*reinterpret_cast<const uint4 *>(tail + ((size_t)b * 4 + 4 + s) * ch + c), v);
        } else if (rev && head) {   // walk step s < 0 of the reverse stream: token len - 1 - s
            unpack8(*reinterpret_cast<const uint4 *>(head + ((size_t)b * 4 - 1 - s) * ch + c), v);
        } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) v[q] = 0.0f;
        }
    };
    if (!conv_w) {
        for (int s = s_begin; s < s_end; ++s) {
            float v[8];
            raw(s, v);
            *reinterpret_cast<uint4 *>(ob + (size_t)s * kBC) = pack8(v);
        }
        return;
    }
    float w0[8], w1[8], w2[8], w3[8], bb[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 t4 = *reinterpret_cast<const float4 *>(conv_w + (size_t)(c + q) * 4);
        w0[q] = t4.x; w1[q] = t4.y; w2[q] = t4.z; w3[q] = t4.w;
        bb[q] = conv_b ? conv_b[c + q] : 0.0f;
    }
    float r0[8], r1[8], r2[8];
    raw(s_begin - 3, r0);
    raw(s_begin - 2, r1);
    raw(s_begin - 1, r2);
    for (int s = s_begin; s < s_end; ++s) {
        float r3[8], o[8];
        raw(s, r3);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float acc = bb[q];
            acc = fmaf(w0[q], r0[q], acc);
            acc = fmaf(w1[q], r1[q], acc);
            acc = fmaf(w2[q], r2[q], acc);
            acc = fmaf(w3[q], r3[q], acc);
            o[q] = tc::silu_tanh(acc);
            r0[q] = r1[q]; r1[q] = r2[q]; r2[q] = r3[q];
        }
        *reinterpret_cast<uint4 *>(ob + (size_t)s * kBC) = pack8(o);
    }
}

// kStateOnly = false: outputs of walk chunks [k0, k0 + nk) of one segment,
// entering it with the state chained from the items before it.
// kStateOnly = true: only the state recurrence over one item's chunks, from a
// zero state; writes the item's end state and its total decay.
// kConcat: untied directions with concatenated outputs; each direction
// stores its own half of every output row and the CTAs never meet.
template <bool kStateOnly, bool kConcat>
__global__ void __launch_bounds__(kThreads, 1)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_x_f, const __grid_constant__ CUtensorMap tm_x_r,
              const __grid_constant__ CUtensorMap tm_bc, const TcParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = tc::smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int hp = blockIdx.x >> 1;          // head pair: heads 2hp, 2hp+1
    const int dir = blockIdx.x & 1;
    const bool rev = dir != 0;
    const int b = blockIdx.y;
    const int H = p.H, L = p.len, ch = p.ch;
    const int HP = H / kHeads;
    const int k0 = blockIdx.z * p.seg_chunks;           // first walk chunk of this CTA
    const int nk = min(p.seg_chunks, p.nchunks - k0);   // walk chunks it covers
    const size_t item_row = ((size_t)(dir * p.batch + b) * HP + hp) * p.nitems;

    float *cum = reinterpret_cast<float *>(sm + kOffCum);   // [chunk parity][head][slot]
    float *dts = reinterpret_cast<float *>(sm + kOffDt);
    float *fB = reinterpret_cast<float *>(sm + kOffFB);
    float *wgt = reinterpret_cast<float *>(sm + kOffWgt);
    float *f4 = reinterpret_cast<float *>(sm + kOffF4);
    float4 *convw = reinterpret_cast<float4 *>(sm + kOffConvW);
    float *convb = reinterpret_cast<float *>(sm + kOffConvB);
    int *flag_slot = reinterpret_cast<int *>(sm + kOffFlag);
    // mbarriers: B/C tiles landed, raw x landed (buffer 0 / 1), G done,
    // M/state ready for the chunk's MMAs, chunk MMAs done, the dt prefix
    // sums of an even / odd walk chunk written (one barrier per buffer, so
    // that the producer may run a chunk ahead without phase aliasing)
    const uint32_t mb_bc = sbase + kOffMbar;
    const uint32_t mb_x0 = sbase + kOffMbar + 8;
    const uint32_t mb_g = sbase + kOffMbar + 24;
    const uint32_t mb_m = sbase + kOffMbar + 32;
    const uint32_t mb_e = sbase + kOffMbar + 40;
    const uint32_t mb_dt0 = sbase + kOffMbar + 48;   // + 8 * (chunk & 1)
    // a chunk's output rows stored (even / odd walk chunk), and the handshake
    // flag the producer then raises for it (null: nothing to publish)
    const uint32_t mb_rows0 = sbase + kOffMbar + 64;
    int **rel_flag = reinterpret_cast<int **>(sm + kOffMbar + 80);
    // phase D of an even / odd walk chunk done: its cum/dts/fB buffer is free
    const uint32_t mb_free0 = sbase + kOffMbar + 96;
    auto dt_ready = [&](int k, uint32_t &mb, uint32_t &parity) {
        mb = mb_dt0 + 8 * (k & 1);
        parity = (k >> 1) & 1;
    };
    auto xbuf_off = [](int k) { return (k & 1) ? kOffXbuf1 : kOffXbuf0; };
    // TMEM regions that alternate between chunks: G(k) and Yd(k) use
    // columns gcol(k) .. +127, M(k) uses mcol(k) .. +127 (the other region)
    auto gcol = [](int k) -> uint32_t { return (k & 1) ? 128u : 0u; };
    auto mcol = [](int k) -> uint32_t { return (k & 1) ? 0u : 128u; };

    auto chunk_of = [&](int k, int &t0, int &cnt, int &s0) {
        const int kg = k0 + k;
        const int c = rev ? p.nchunks - 1 - kg : kg;
        t0 = c * kQ;
        cnt = min(kQ, L - t0);
        s0 = rev ? L - t0 - cnt : t0;
        return c;
    };
    // raw x rows of chunk k (+ conv halo) into x buffer k % 2
    auto issue_x = [&](int k) {
        int t0, cnt, s0;
        chunk_of(k, t0, cnt, s0);
        const uint32_t mb = mb_x0 + 8 * (k & 1);
        tc::mbar_expect_tx(mb, kRawBytes);
        tc::tma_load_3d(sbase + xbuf_off(k), rev ? &tm_x_r : &tm_x_f, hp * kPP, rev ? t0 : t0 - 3, b,
                        mb);
    };
    auto issue_bc = [&](int k) {
        int t0, cnt, s0;
        chunk_of(k, t0, cnt, s0);
        const int zc = dir * p.batch + b;
        tc::mbar_expect_tx(mb_bc, kStateOnly ? kBCBytes / 2 : kBCBytes);
        tc::tma_load_3d(sbase + kOffB, &tm_bc, 0, s0, zc, mb_bc);
        tc::tma_load_3d(sbase + kOffB + 16384, &tm_bc, 64, s0, zc, mb_bc);
        if constexpr (!kStateOnly) {
            tc::tma_load_3d(sbase + kOffC, &tm_bc, 128, s0, zc, mb_bc);
            tc::tma_load_3d(sbase + kOffC + 16384, &tm_bc, 192, s0, zc, mb_bc);
        }
    };

    constexpr float kLog2e = 1.4426950408889634f;
    const float *Adir = rev ? p.A[1] : p.A[0];
    const float A0 = Adir[hp * kHeads] * kLog2e, A1 = Adir[hp * kHeads + 1] * kLog2e;

    // helper warp: asynchronous copy of walk chunk k's dt (both heads of
    // the pair are adjacent: one 4-byte copy per token) into dt buffer
    // k % 2; slots past the chunk end are zero.
    auto load_dt_async = [&](int k) {
        int t0, cnt, s0;
        chunk_of(k, t0, cnt, s0);
        uint32_t *dst = reinterpret_cast<uint32_t *>(sm + kOffDtBuf) + (k & 1) * kQ;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int j = 4 * lane + i;
            if (j < cnt) {
                const int s = s0 + j;
                const int tok = rev ? L - 1 - s : s;
                const __nv_bfloat16 *src = (rev ? p.dt[1] : p.dt[0]) + ((size_t)b * L + tok) * H + hp * kHeads;
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;"
                             :: "r"(tc::smem_u32(dst + j)), "l"(src) : "memory");
            } else {
                dst[j] = 0u;
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // helper warp: inclusive prefix sums of dt*A of both heads for walk
    // chunk k into cum/dts buffer k % 2, in log2 units (A carries the factor
    // log2(e)) so that every decay factor is one 2^x on the special-function
    // unit, then the chunk's per-slot factors.  Waits for this thread's
    // outstanding dt copies (chunk k's and, if issued, chunk k+1's).
    auto scan_dt = [&](int k) {
        asm volatile("cp.async.wait_all;" ::: "memory");
        const __nv_bfloat162 *src =
            reinterpret_cast<const __nv_bfloat162 *>(sm + kOffDtBuf) + (k & 1) * kQ + 4 * lane;
#pragma unroll
        for (int head = 0; head < kHeads; ++head) {
            float d[4], a[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(src[i]);
                d[i] = head ? f.y : f.x;
            }
            const float Aw = head ? A1 : A0;
            a[0] = d[0] * Aw;
#pragma unroll
            for (int i = 1; i < 4; ++i) a[i] = fmaf(d[i], Aw, a[i - 1]);
            float run = a[3];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float v = __shfl_up_sync(0xffffffffu, run, o);
                if (lane >= o) run += v;
            }
            const float excl = run - a[3];
            float *db = dts + ((k & 1) * kHeads + head) * kQ + 4 * lane;
            float *cb = cum + ((k & 1) * kHeads + head) * kQ + 4 * lane;
            *reinterpret_cast<float4 *>(db) = make_float4(d[0], d[1], d[2], d[3]);
            *reinterpret_cast<float4 *>(cb) =
                make_float4(excl + a[0], excl + a[1], excl + a[2], excl + a[3]);
        }
        // per-slot decay factors, from the sums the other lanes just wrote:
        // w = exp(c_last - c_s) dt_s, fB = exp(c_R - c_s) dt_s (R = end of
        // s's 32-slot block) and f4 = exp(c_R4 - c_s) dt_s (R4 = s | 3)
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kHeads * kQ / 32; ++i) {
            const int e = (k & 1) * kHeads * kQ + 32 * i + lane;   // [parity][head][slot]
            const float cs = cum[e];
            const float d = dts[e];
            wgt[e] = tc::exp2_approx(cum[e | (kQ - 1)] - cs) * d;
            if constexpr (!kStateOnly) {   // M's factors; the state-only pass needs w only
                fB[e] = tc::exp2_approx(cum[e | 31] - cs) * d;
                f4[e] = tc::exp2_approx(cum[e | 3] - cs) * d;
            }
        }
    };

    // ---- setup (all threads)
    const float *conv_w = rev ? p.conv_w[1] : p.conv_w[0];
    const float *conv_b = rev ? p.conv_b[1] : p.conv_b[0];
    const bool has_conv = conv_w != nullptr;
    if (tid < kPP && has_conv) {
        // stored as [q][g] for local channel 8g + q, so that the 16 channel
        // groups of a warp read 16 consecutive entries (no bank conflicts)
        const int c = hp * kPP + tid;
        const int slot = (tid & 7) * (kPP / 8) + (tid >> 3);
        convw[slot] = *reinterpret_cast<const float4 *>(conv_w + (size_t)c * 4);
        convb[slot] = conv_b ? conv_b[c] : 0.0f;
    }
    if (warp == 0) tc::tmem_alloc(sbase + kOffTmem, kTmemCols);
    if (tid == kProducerTid) {
        tc::prefetch_tmap(rev ? &tm_x_r : &tm_x_f);
        tc::prefetch_tmap(&tm_bc);
        tc::mbar_init(mb_bc, 1);
        tc::mbar_init(mb_x0, 1);
        tc::mbar_init(mb_x0 + 8, 1);
        tc::mbar_init(mb_g, 1);
        tc::mbar_init(mb_m, 1);
        tc::mbar_init(mb_e, 1);
        tc::mbar_init(mb_dt0, 32);       // every helper lane arrives after its part of a scan
        tc::mbar_init(mb_dt0 + 8, 32);
        tc::mbar_init(mb_free0, 1);
        tc::mbar_init(mb_free0 + 8, 1);
        tc::mbar_init(mb_rows0, 1);
        tc::mbar_init(mb_rows0 + 8, 1);
        issue_x(0);
        if (nk > 1) issue_x(1);
        issue_bc(0);
    }
    // Global loads that need nothing from the set-up start before its
    // barrier, so that their latencies overlap (they dominate a CTA that
    // covers a single chunk, as in block decode): the helper's first dt
    // copies, and each compute thread's share of the caller's initial state.
    if (warp == kHelperWarp) {
        load_dt_async(0);
        if (nk > 1) load_dt_async(1);
    }
    float sv_init[32];
    {
        const int row = tid & 127, rg = tid >> 7;
        const size_t sidx0 = ((size_t)b * H + hp * kHeads + (rg >> 1)) * kP * kN;
        const bool use_init = !kStateOnly && !rev && p.init && tid < kAluThreads;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            sv_init[i] = use_init ? __ldg(p.init + sidx0 + (size_t)(32 * (rg & 1) + i) * kN + row) : 0.0f;
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kOffTmem);

    if (warp == kProducerWarp) {
        // ================= producer: every MMA and every TMA load, and the
        // release of each chunk's rows (lane 0)
        const uint64_t dC = tc::smem_desc(sbase + kOffC, 16, 1024);       // K-major A (G, Yo)
        const uint64_t dB = tc::smem_desc(sbase + kOffB, 16, 1024);       // K-major B (G)
        const uint64_t dBmn = tc::smem_desc(sbase + kOffB, 16384, 1024);  // MN-major A (state)
        const uint64_t dX0 = tc::smem_desc(sbase + kOffXbuf0, 1024, 1024);  // MN-major B (Yd)
        const uint64_t dX1 = tc::smem_desc(sbase + kOffXbuf1, 1024, 1024);
        const uint64_t dS = tc::smem_desc(sbase + kOffS, 16384, 1024);    // MN-major B (Yo)
        const uint64_t dXw = tc::smem_desc(sbase + kOffXw, 16384, 1024);  // MN-major B (state)
        constexpr uint32_t idG = tc::idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idYd = tc::idesc_bf16(128, 64, 0, 1);
        constexpr uint32_t idYo = tc::idesc_bf16(128, 128, 0, 1);
        constexpr uint32_t idS = tc::idesc_bf16(128, 128, 1, 1);
        // lane 0: once chunk j's rows are stored, publish them to the partner
        // CTA if this CTA arrived first (GPU-scope release; the rows were
        // made visible to this thread through the group barrier and the
        // mbarrier).  Done here so that the compute group never waits on it.
        auto release_rows = [&](int j) -> bool {
            const bool w = tc::mbar_wait_bounded(mb_rows0 + 8 * (j & 1), (j >> 1) & 1, kWaitCycles);
            if (w) {
                int *f = rel_flag[j & 1];
                if (f) st_release(f, 1);
            }
            return w;
        };
        bool pok = true;
        for (int k = 0; k < nk && pok; ++k) {
            const uint32_t g = tmem + gcol(k);
            if (lane == 0) {
                // G(k) overwrites region gcol(k), last used by M(k-1): wait
                // for the MMAs of chunk k-1, and for this chunk's B/C tiles
                if (!kStateOnly && k > 0) pok = tc::mbar_wait_bounded(mb_e, (k - 1) & 1, kWaitCycles);
                if (pok) pok = tc::mbar_wait_bounded(mb_bc, k & 1, kWaitCycles);
                if (pok) {
                    tc::fence_after_sync();
                    if constexpr (!kStateOnly) {
#pragma unroll
                        for (int ks = 0; ks < kN / 16; ++ks) {
                            const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                            tc::mma_bf16(g, tc::desc_add(dC, koff), tc::desc_add(dB, koff), idG, ks > 0);
                        }
                        tc::mma_commit(mb_g);
                    }
                }
            }
            if (lane == 0) {
                if (!kStateOnly && k > 0 && pok) pok = release_rows(k - 1);
                // Yd_h = M_h X_h, Yo = C S_in^T, S^T += B^T (wX)
                if (pok) pok = tc::mbar_wait_bounded(mb_m, k & 1, kWaitCycles);
                if (pok) {
                    tc::fence_after_sync();
                    if constexpr (!kStateOnly) {
                        const uint64_t dX = (k & 1) ? dX1 : dX0;
                        const uint32_t mc = tmem + mcol(k);
#pragma unroll
                        for (int ks = 0; ks < kQ / 16; ++ks) {
#pragma unroll
                            for (int hd = 0; hd < kHeads; ++hd)
                                tc::mma_bf16_tmemA(g + 64 * hd, mc + 64 * hd + 8 * ks,
                                                   tc::desc_add(dX, hd * 16384 + ks * 2048), idYd, ks > 0);
                        }
                    }
#pragma unroll
                    for (int ks = 0; ks < kN / 16; ++ks) {
                        const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                        if constexpr (!kStateOnly)
                            tc::mma_bf16(tmem + kColYo, tc::desc_add(dC, koff), tc::desc_add(dS, ks * 2048),
                                         idYo, ks > 0);
                        tc::mma_bf16(tmem + kColS, tc::desc_add(dBmn, ks * 2048),
                                     tc::desc_add(dXw, ks * 2048), idS, 1);
                    }
                    tc::mma_commit(mb_e);
                }
            }
            pok = __shfl_sync(0xffffffffu, pok, 0);
            if (!pok || k + 1 >= nk) break;
            // once they complete, the B/C tiles and this chunk's x buffer
            // are free: load the next chunk's tiles and the chunk after
            // next's raw x rows
            if (lane == 0) {
                pok = tc::mbar_wait_bounded(mb_e, k & 1, kWaitCycles);
                if (pok) {
                    issue_bc(k + 1);
                    if (k + 2 < nk) issue_x(k + 2);
                }
            }
            pok = __shfl_sync(0xffffffffu, pok, 0);
        }
        if (!kStateOnly && lane == 0 && pok && nk > 0) pok = release_rows(nk - 1);
        if (lane == 0 && !pok) record_error(p.status, kStatusTimeout);
    } else if (warp == kHelperWarp) {
        // ================= helper: dt copies, prefix sums and slot factors
        // of each chunk, up to two chunks ahead of phase D (the copies of
        // chunks 0 and 1 were issued before the set-up barrier)
        bool hok = true;
        for (int j = 0; j < nk; ++j) {
            if (j >= 2) {
                // buffer j % 2 last held chunk j-2, read up to its phase D
                if (lane == 0)
                    hok = tc::mbar_wait_bounded(mb_free0 + 8 * (j & 1), ((j >> 1) - 1) & 1, kWaitCycles);
                hok = __shfl_sync(0xffffffffu, hok, 0);
                if (!hok) break;
            }
            scan_dt(j);
            if (j + 2 < nk) load_dt_async(j + 2);
            tc::mbar_arrive(mb_dt0 + 8 * (j & 1));
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
        if (lane == 0 && !hok) record_error(p.status, kStatusTimeout);
    } else {
        // ================= compute group: 512 threads ======================
        // thread roles: row = TMEM lane / tile row; rg = 32-column group of
        // the head pair's 128 columns (head rg >> 1, half rg & 1)
        const int row = tid & 127;
        const int rg = tid >> 7;
        const int hh = rg >> 1;
        const int hsub = rg & 1;
        const uint32_t lane_base = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const int quad = warp & 3;
        // conv+SiLU of both heads' x for walk chunk k, in place: the raw
        // rows in x buffer k % 2 become the swizzled X tile of the chunk.
        // Thread: 8 channels (group g: head g >> 3, piece g & 7) x 4 slots.
        // Raw row of token u: forward u - (t0 - 3), reverse u - t0.  Every
        // thread reads its raw rows before the barrier and writes after it.
        auto conv_chunk = [&](int k) {
            int t0, cnt, s0;
            chunk_of(k, t0, cnt, s0);
            uint8_t *buf = sm + xbuf_off(k);
            const __nv_bfloat16 *rawp = reinterpret_cast<const __nv_bfloat16 *>(buf);
            const int g = tid & 15;
            const int gh = g >> 3, gp = g & 7;
            const int j0 = (tid >> 4) * 4;
            uint4 rr[7];
#pragma unroll
            for (int i = 0; i < 7; ++i) {
                const int jw = j0 + i - 3;   // walk offset of the raw row
                const int rrow = rev ? cnt - 1 - jw : jw + 3;
                rr[i] = (rrow >= 0 && rrow < kRawRows)
                            ? *reinterpret_cast<const uint4 *>(rawp + rrow * kPP + 8 * g)
                            : make_uint4(0, 0, 0, 0);
            }
            alu_sync();
            float o[4][8];
            const __nv_bfloat16 *ru = reinterpret_cast<const __nv_bfloat16 *>(rr);
            if (has_conv) {
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const float4 w4 = convw[q * (kPP / 8) + g];
                    const float bq = convb[q * (kPP / 8) + g];
                    float u[7];
#pragma unroll
                    for (int r = 0; r < 7; ++r) u[r] = __bfloat162float(ru[8 * r + q]);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        float acc = bq;
                        acc = fmaf(w4.x, u[i], acc);
                        acc = fmaf(w4.y, u[i + 1], acc);
                        acc = fmaf(w4.z, u[i + 2], acc);
                        acc = fmaf(w4.w, u[i + 3], acc);
                        o[i][q] = (j0 + i < cnt) ? tc::silu_tanh(acc) : 0.0f;
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        o[i][q] = (j0 + i < cnt) ? __bfloat162float(ru[8 * (i + 3) + q]) : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<uint4 *>(buf + gh * 16384 + tc::sw128(j0 + i, gp)) = pack8(o[i]);
        };
        // wX = w_s * X for walk chunk k (X tile in x buffer k % 2)
        auto weight_chunk = [&](int k) {
            const uint8_t *xt = sm + xbuf_off(k);
            const int j = tid & 127, q4 = tid >> 7;   // slot, quarter of the 128 columns
            const int gh = q4 >> 1;
            const float wj = wgt[((k & 1) * kHeads + gh) * kQ + j];
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
                const uint32_t off = gh * 16384 + tc::sw128(j, 4 * (q4 & 1) + pc);
                float v[8];
                unpack8(*reinterpret_cast<const uint4 *>(xt + off), v);
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] *= wj;
                *reinterpret_cast<uint4 *>(sm + kOffXw + off) = pack8(v);
            }
        };
        // one thread polls an mbarrier (two if mb2 != 0); the group barrier
        // releases the rest
        auto wait_all = [&](uint32_t mb, uint32_t parity, uint32_t mb2 = 0, uint32_t parity2 = 0) -> bool {
            bool w = true;
            if (tid == 0) {
                w = tc::mbar_wait_bounded(mb, parity, kWaitCycles);
                if (w && mb2) w = tc::mbar_wait_bounded(mb2, parity2, kWaitCycles);
            }
            return alu_sync_and(w);
        };

        // ---- state S^T[n = row][p' = 32*rg + i] -> TMEM columns kColS + 32*rg.
        // A segment's entering state: the caller's initial state (forward
        // stream; loaded before the set-up barrier) or zero, carried through
        // the items before the segment: S <- 2^dec_i S + S_i, with S_i item
        // i's end state from zero.
        const int head_g = hp * kHeads + hh;     // global head of this thread's columns
        const size_t sidx = ((size_t)b * H + head_g) * kP * kN;
        {
            float sv[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) sv[i] = sv_init[i];
            // sequence shards: the walk enters this shard with the state the
            // shards before it in walk order leave (forward: ranks 0..rank-1
            // from the initial state; reverse: ranks nranks-1..rank+1 from zero)
            const int n_sh = (kStateOnly || !p.shard_states) ? 0 : (rev ? p.nranks - 1 - p.rank : p.rank);
            for (int it = 0; it < n_sh; ++it) {
                const int q = rev ? p.nranks - 1 - it : it;
                const size_t e = (((size_t)q * 2 + dir) * p.batch + b) * H + head_g;
                const float *si = p.shard_states + e * kP * kN;
                const float a = tc::exp2_approx(p.shard_dec[e]);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = fmaf(sv[i], a, si[(size_t)(32 * hsub + i) * kN + row]);
            }
            const int n_in = (kStateOnly || p.item_chunks == 0) ? 0 : k0 / p.item_chunks;
            for (int it = 0; it < n_in; ++it) {
                const float *si = p.seg_state + ((item_row + it) * kHeads + hh) * kP * kN;
                const float a = tc::exp2_approx(p.seg_dec[(item_row + it) * kHeads + hh]);
#pragma unroll
                for (int i = 0; i < 32; ++i) sv[i] = fmaf(sv[i], a, si[(size_t)(32 * hsub + i) * kN + row]);
            }
#pragma unroll
            for (int half16 = 0; half16 < 2; ++half16) {
                uint32_t r[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(sv[16 * half16 + i]);
                tc::tmem_st16(tmem + lane_base + kColS + 32 * rg + 16 * half16, r);
            }
        }
        uint32_t mbd, pard;
        dt_ready(0, mbd, pard);
        bool ok = wait_all(mbd, pard);   // chunk 0's prefix sums and slot factors
        float dec = 0.0f;   // state-only: total decay of the item (log2 units)
        const float Dh = kStateOnly ? 0.0f : (rev ? p.D[1] : p.D[0])[head_g];   // no D for states

        int arrival = 0;   // result of this chunk's arrival atomic (thread kArriveTid)
        ok = ok && wait_all(mb_x0, 0);
        if (ok) {
            // decode and sequence shards: the conv history before token 0
            // comes from the tail; for sequence shards the reverse stream's
            // conv reads the tokens after the shard from the head (raw rows
            // cnt .. cnt+2 of the walk's first chunk, past the shard end)
            if (!rev && p.tail && k0 == 0) {
                for (int e = tid; e < 3 * (kPP / 8); e += kAluThreads) {
                    const int r = e / (kPP / 8), g = e % (kPP / 8);
                    *reinterpret_cast<uint4 *>(sm + kOffXbuf0 + r * (kPP * 2) + g * 16) =
                        *reinterpret_cast<const uint4 *>(p.tail + ((size_t)b * 4 + 1 + r) * ch +
                                                         hp * kPP + 8 * g);
                }
                alu_sync();
            }
            if (rev && p.head && k0 == 0) {
                int t0, cnt, s0;
                chunk_of(0, t0, cnt, s0);
                for (int e = tid; e < 3 * (kPP / 8); e += kAluThreads) {
                    const int r = e / (kPP / 8), g = e % (kPP / 8);
                    *reinterpret_cast<uint4 *>(sm + kOffXbuf0 + (cnt + r) * (kPP * 2) + g * 16) =
                        *reinterpret_cast<const uint4 *>(p.head + ((size_t)b * 4 + r) * ch +
                                                         hp * kPP + 8 * g);
                }
                alu_sync();
            }
            conv_chunk(0);
            alu_sync();
            weight_chunk(0);
        }

        for (int k = 0; k < nk && ok; ++k) {
            int t0, cnt, s0;
            const int c = chunk_of(k, t0, cnt, s0);
            const bool more = k + 1 < nk;

            // arrive at this chunk's forward/reverse meeting point; the
            // result is read only after the chunk's MMAs
            if (!kStateOnly && !kConcat && tid == kArriveTid)
                arrival = atomicAdd(p.flags + (((size_t)b * HP + hp) * p.nchunks + c) * 2, 1);

            // ---- D: M_h (both heads, into TMEM) and the state's chunk-start
            // scaling, once G(k) is done.  Thread (row t, rg): head hh,
            // s-blocks 2*hsub, 2*hsub+1.
            tc::fence_proxy_async();          // wX of this chunk (written last iteration)
            if constexpr (!kStateOnly) {
                ok = wait_all(mb_g, k & 1);
                if (!ok) break;
            }
            tc::fence_after_sync();
            const float *cumk = cum + ((k & 1) * kHeads + hh) * kQ;   // this chunk, this head
            const float *dtsk = dts + ((k & 1) * kHeads + hh) * kQ;
            const float ct = cumk[row];                     // kept for the epilogue
            const float a_last = tc::exp2_approx(cumk[kQ - 1]);
            if constexpr (kStateOnly) dec += cumk[kQ - 1];
            {
                const uint32_t gc = gcol(k), mc = mcol(k);
                if constexpr (!kStateOnly) {
#pragma unroll
                    for (int jj = 0; jj < 2; ++jj) {
                        const int jb = 2 * hsub + jj;           // 32-slot block of s
                        uint32_t packed[16];
                        if (jb > quad) {                        // warp-uniform: all s > t
#pragma unroll
                            for (int i = 0; i < 16; ++i) packed[i] = 0u;
                        } else {
                            float gv[32];
                            tc::tmem_ld32(tmem + lane_base + gc + 32 * jb, gv);
                            const float *fbh = fB + ((k & 1) * kHeads + hh) * kQ + 32 * jb;
                            if (jb < quad) {
                                // whole block below the diagonal: factorised decay
                                const float et = tc::exp2_approx(ct - cumk[32 * jb + 31]);
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    packed[i] = tc::pack_bf16x2(gv[2 * i] * et * fbh[2 * i],
                                                                gv[2 * i + 1] * et * fbh[2 * i + 1]);
                            } else {
                                // diagonal block, D on the diagonal
                                const float *ch_ = cumk + 32 * jb;
                                const int r31 = row & 31;
                                if (ch_[0] - ch_[31] <= 60.0f) {   // warp-uniform (head, block)
                                    // 4-slot sub-blocks: exp(c_t - c_s) = exp(c_t - c_R4)
                                    // exp(c_R4 - c_s), R4 = s | 3.  With the block's whole
                                    // decay at most 2^60 neither factor overflows; for s <= t
                                    // the product is the decay itself
                                    const float *f4h = f4 + ((k & 1) * kHeads + hh) * kQ + 32 * jb;
                                    float rf[8];
#pragma unroll
                                    for (int j = 0; j < 8; ++j) rf[j] = tc::exp2_approx(ct - ch_[4 * j + 3]);
#pragma unroll
                                    for (int i = 0; i < 32; ++i) {
                                        const float v = fmaf(gv[i] * rf[i >> 2], f4h[i], (i == r31) ? Dh : 0.0f);
                                        gv[i] = (i <= r31) ? v : 0.0f;
                                    }
                                } else {
                                    // steep decays: one exponential per element, each <= 1
                                    const float *dh_ = dtsk + 32 * jb;
#pragma unroll
                                    for (int i = 0; i < 32; ++i) {
                                        const float e = tc::exp2_approx(fminf(ct - ch_[i], 0.0f));
                                        const float v = fmaf(gv[i] * e, dh_[i], (i == r31) ? Dh : 0.0f);
                                        gv[i] = (i <= r31) ? v : 0.0f;
                                    }
                                }
#pragma unroll
                                for (int i = 0; i < 16; ++i) packed[i] = tc::pack_bf16x2(gv[2 * i], gv[2 * i + 1]);
                            }
                        }
                        tc::tmem_st16(tmem + lane_base + mc + 64 * hh + 16 * jb, packed);
                    }
                }
                // state: bf16 copy of S_in (the Yo operand), then S <- exp(c_last) S
                float sv[32];
                tc::tmem_ld32(tmem + lane_base + kColS + 32 * rg, sv);
                if constexpr (!kStateOnly) {
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc)
                        *reinterpret_cast<uint4 *>(sm + kOffS + hh * 16384 +
                                                   tc::sw128(row, 4 * hsub + pc)) = pack8(sv + 8 * pc);
                }
#pragma unroll
                for (int half16 = 0; half16 < 2; ++half16) {
                    uint32_t r[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(sv[16 * half16 + i] * a_last);
                    tc::tmem_st16(tmem + lane_base + kColS + 32 * rg + 16 * half16, r);
                }
            }
            tc::fence_proxy_async();
            tc::fence_before_sync();
            alu_sync();
            if (tid == 0) {
                tc::mbar_arrive(mb_m);                  // the producer issues the MMAs
                tc::mbar_arrive(mb_free0 + 8 * (k & 1));   // the helper may reuse this chunk's buffers
            }

            // ---- while the MMAs run: the next chunk's conv
            if (more) {
                ok = wait_all(mb_x0 + 8 * ((k + 1) & 1), ((k + 1) >> 1) & 1);
                if (!ok) break;
                conv_chunk(k + 1);
            }
            if (!kStateOnly && tid == kArriveTid) *flag_slot = arrival;
            // the chunk's MMAs done, and (helper) the next chunk's prefix sums
            // and slot factors
            dt_ready(k + 1, mbd, pard);
            ok = more ? wait_all(mb_e, k & 1, mbd, pard) : wait_all(mb_e, k & 1);
            if (!ok) break;
            tc::fence_after_sync();
            if constexpr (kStateOnly) {
                if (more) weight_chunk(k + 1);
                continue;
            }

            // ---- F: output rows, and the forward + reverse sum
            int *fl = p.flags + (((size_t)b * HP + hp) * p.nchunks + c) * 2;
            const bool first = *flag_slot == 0;
            bool ready = true;
            if (!first && tid == 0) {
                // the partner CTA arrived first; wait (bounded) until its
                // output is visible
                ready = ld_acquire(fl + 1) != 0;
                if (!ready) {
                    const long long w0 = clock64();
                    while (!(ready = ld_acquire(fl + 1) != 0)) {
                        if (clock64() - w0 > kWaitCycles) break;
                    }
                }
            }
            // releases the group after thread 0's wait for the partner.  A
            // wait that gave up stops the walk here: the partner's rows are
            // not added to, and the meeting counters are left as they are
            // (the caller zero-fills the workspace again after a timeout).
            if (!alu_sync_and(ready)) {
                ok = false;
                break;
            }
            // the next chunk's wX first, while the partner's rows can be fetched
            if (more) weight_chunk(k + 1);
            // Coalesced output: each thread stages its 32 outputs in shared
            // memory (the bf16 state copy's buffer, free until the next
            // chunk's phase D), then 16 threads per token row move whole
            // 256-byte rows.  Staging layout: [t][16 pieces of 16 B], piece
            // q of row t stored at q ^ (t & 15) (conflict-free both ways).
            const int cp = tid & 15;          // 16-byte piece of a row (8 channels)
            const int cr = tid >> 4;          // rows cr, cr+32, cr+64, cr+96
            auto ypiece = [&](int r) -> uint4 * {
                const int tk = rev ? t0 + cnt - 1 - r : t0 + r;
                const size_t row0 = kConcat ? ((size_t)b * L + tk) * 2 * H * kP + dir * H * kP
                                            : ((size_t)b * L + tk) * H * kP;
                return reinterpret_cast<uint4 *>(p.y + row0 + hp * kPP) + cp;
            };
            {
                float yd[32], yo[32];
                tc::tmem_ld32(tmem + lane_base + gcol(k) + 64 * hh + 32 * hsub, yd);
                tc::tmem_ld32(tmem + lane_base + kColYo + 64 * hh + 32 * hsub, yo);
                const float et = tc::exp2_approx(ct);
#pragma unroll
                for (int i = 0; i < 32; ++i) yd[i] = fmaf(et, yo[i], yd[i]);
#pragma unroll
                for (int pc = 0; pc < 4; ++pc)
                    *reinterpret_cast<uint4 *>(sm + kOffS + row * 256 +
                                               (((4 * rg + pc) ^ (row & 15)) << 4)) = pack8(yd + 8 * pc);
            }
            tc::fence_before_sync();
            alu_sync();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = cr + 32 * j;
                if (r < cnt) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(sm + kOffS + r * 256 +
                                                                     ((cp ^ (r & 15)) << 4));
                    if (first) {
                        *ypiece(r) = v;
                    } else {
                        // second to reach the chunk: add to the partner's rows
                        // at L2 (bf16 reductions, ordered after the partner's
                        // release through thread 0's acquire and the barrier)
                        asm volatile("red.global.add.noftz.v4.bf16x2 [%0], {%1, %2, %3, %4};"
                                     :: "l"(ypiece(r)), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                                     : "memory");
                    }
                }
            }
            alu_sync();   // rows stored; the staging buffer is rewritten by the next chunk's phase D
            if (tid == 0) {
                if (!first) {
                    fl[0] = 0;   // leave the workspace zeroed for the next call
                    fl[1] = 0;
                }
                rel_flag[k & 1] = (first && !kConcat) ? fl + 1 : nullptr;
                tc::mbar_arrive(mb_rows0 + 8 * (k & 1));   // the producer publishes them
            }
        }

        if constexpr (kStateOnly) {
            if (ok) {
                // the item's end state and total decay
                tc::fence_after_sync();
                float sv[32];
                tc::tmem_ld32(tmem + lane_base + kColS + 32 * rg, sv);
                const size_t item = item_row + blockIdx.z;
                float *so = p.seg_state + (item * kHeads + hh) * kP * kN;
#pragma unroll
                for (int i = 0; i < 32; ++i) so[(size_t)(32 * hsub + i) * kN + row] = sv[i];
                if (row == 0 && hsub == 0) p.seg_dec[item * kHeads + hh] = dec;
            }
        } else if (ok && !rev && p.fin && k0 + nk == p.nchunks) {
            tc::fence_after_sync();
            float sv[32];
            tc::tmem_ld32(tmem + lane_base + kColS + 32 * rg, sv);
#pragma unroll
            for (int i = 0; i < 32; ++i) p.fin[sidx + (size_t)(32 * hsub + i) * kN + row] = sv[i];
        }
        if (!ok && tid == 0) record_error(p.status, kStatusTimeout);
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

bool tc_path_supported(const bimamba_dims &d)
{
    return d.dtype == BIMAMBA_BF16 && d.headdim == kP && d.d_state == kN && d.ngroups == 1 &&
           d.d_conv == 4 && d.len > 0 && d.heads % kHeads == 0;
}

// Segments.  One CTA per (batch, head pair, direction) fills the 148 SMs
// only when batch * heads >= 148.  Otherwise each direction's walk is cut
// into nseg segments of seg_chunks chunks, run side by side.  A segment must
// start from the state the walk carries into it, so a state-only pass first
// reduces each of the nitems = (nseg - 1) * r items (seg_chunks / r chunks
// each) before the last segment to its end state from zero and its total
// decay; a segment's CTA then chains the items before it (the recurrence is
// linear in the state, so S_in = 2^dec_i S_in + S_i over the items in order).
// r > 1 splits the state-only pass finer than the segments, so that it too
// fills the SMs.
struct SegPlan {
    int nseg, seg_chunks, item_chunks, nitems;
};

constexpr int kPlanSMs = 148;   // SMs of a B200

static SegPlan seg_plan(const bimamba_dims &d)
{
    const int nchunks = (int)(((long long)d.len + kQ - 1) / kQ);
    const SegPlan whole{1, nchunks, 0, 0};
    const long long ctas = (long long)d.heads * d.batch;   // head pairs x 2 directions
    if (ctas <= 0 || ctas * 2 > kPlanSMs || nchunks < 4) return whole;
    const int nseg_target = (int)(kPlanSMs / ctas);
    const int r = (int)std::max<long long>(1, kPlanSMs / (ctas * (nseg_target - 1)));
    const int item_chunks = (nchunks + nseg_target * r - 1) / (nseg_target * r);
    const int seg_chunks = r * item_chunks;
    const int nseg = (nchunks + seg_chunks - 1) / seg_chunks;
    if (nseg < 2) return whole;
    return SegPlan{nseg, seg_chunks, item_chunks, (nseg - 1) * r};
}

// workspace: [flags: batch*(H/2)*nchunks*2 int32, 1 KB aligned][B/C activations:
// 2 directions x batch x len x 256 bf16][item states: 2 x batch x H/2 x nitems
// x 2 x kP x kN f32][item decays: 2 x batch x H/2 x nitems x 2 f32]
static size_t flags_bytes(const bimamba_dims &d)
{
    const size_t nchunks = ((size_t)d.len + kQ - 1) / kQ;
    const size_t bytes = (size_t)d.batch * (d.heads / kHeads) * nchunks * 2 * sizeof(int);
    return (bytes + 1023) & ~(size_t)1023;
}

static size_t act_bytes(const bimamba_dims &d)
{
    return (size_t)2 * d.batch * d.len * kBC * sizeof(__nv_bfloat16);
}

static size_t items(const bimamba_dims &d, const SegPlan &sp)
{
    return (size_t)2 * d.batch * (d.heads / kHeads) * sp.nitems;
}

void tc_launch_plan(const bimamba_dims &d, int *out)
{
    const SegPlan sp = seg_plan(d);
    out[0] = sp.nseg;
    out[1] = sp.seg_chunks;
    out[2] = sp.nitems;
}

size_t tc_counter_bytes(const bimamba_dims &d) { return flags_bytes(d); }

size_t tc_workspace_bytes(const bimamba_dims &d)
{
    const SegPlan sp = seg_plan(d);
    const size_t n = items(d, sp);
    return flags_bytes(d) + act_bytes(d) + n * kHeads * kP * kN * sizeof(float) +
           n * kHeads * sizeof(float);
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    }
    return fn;
}

// 3-D bf16 tensor map: dims (inner, rows, planes), box (box0, box1, 1).
static bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows,
                     uint64_t planes, uint32_t box0, uint32_t box1, bool swizzle128)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {inner, rows, planes};
    const cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
    const cuuint32_t box[3] = {box0, box1, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_shard_states(const Problem &pr, cudaStream_t stream)
{
    return launch_ssd_tc(pr, stream);   // pr.states_out selects the states-only launch
}

cudaError_t launch_ssd_tc(const Problem &pr, cudaStream_t stream)
{
    const bimamba_dims &d = pr.dims;
    TcParams p;
    const __nv_bfloat16 *xbc[2];
    for (int i = 0; i < 2; ++i) {
        xbc[i] = static_cast<const __nv_bfloat16 *>(pr.xbc[i]);
        p.dt[i] = static_cast<const __nv_bfloat16 *>(pr.dt[i]);
        p.A[i] = pr.A[i];
        p.D[i] = pr.D[i];
        p.conv_w[i] = pr.conv_w[i];
        p.conv_b[i] = pr.conv_b[i];
    }
    p.tail = static_cast<const __nv_bfloat16 *>(pr.tail);
    p.head = static_cast<const __nv_bfloat16 *>(pr.head);
    p.shard_states = pr.shard_states;
    p.shard_dec = pr.shard_dec;
    p.rank = pr.rank;
    p.nranks = pr.nranks;
    p.init = pr.init;
    p.fin = pr.fin;
    p.y = static_cast<__nv_bfloat16 *>(pr.y);

    p.flags = static_cast<int *>(pr.workspace);
    p.status = pr.status;
    p.len = d.len;
    p.H = d.heads;
    p.ch = d.heads * d.headdim + 2 * d.ngroups * d.d_state;
    p.nchunks = (d.len + kQ - 1) / kQ;
    p.batch = d.batch;
    char *ws = static_cast<char *>(pr.workspace);
    __nv_bfloat16 *act = reinterpret_cast<__nv_bfloat16 *>(ws + flags_bytes(d));
    const SegPlan sp = seg_plan(d);
    const size_t n_items = items(d, sp);
    p.seg_state = reinterpret_cast<float *>(ws + flags_bytes(d) + act_bytes(d));
    p.seg_dec = p.seg_state + n_items * kHeads * kP * kN;
    p.seg_chunks = sp.seg_chunks;
    p.item_chunks = sp.item_chunks;
    p.nitems = sp.nitems;

    // prepass: B/C conv+SiLU in walk order for both directions
    bc_prepass_kernel<<<dim3((d.len + 31) / 32, d.batch, 2), 128, 0, stream>>>(
        xbc[0], xbc[1], p.tail, p.head, p.conv_w[0], p.conv_w[1], p.conv_b[0], p.conv_b[1], act, d.len,
        p.ch, d.heads * kP, d.batch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();

    CUtensorMap tm_x_f, tm_x_r, tm_bc;
    if (!make_map(&tm_x_f, xbc[0], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, kPP, kRawRows,
                  false) ||
        !make_map(&tm_x_r, xbc[1], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, kPP, kRawRows,
                  false) ||
        !make_map(&tm_bc, act, (uint64_t)kBC, (uint64_t)d.len, (uint64_t)2 * d.batch, 64, kQ, true))
        return cudaErrorInvalidValue;
    auto main_kernel = pr.concat ? ssd_tc_kernel<false, true> : ssd_tc_kernel<false, false>;
    e = cudaFuncSetAttribute(main_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ssd_tc_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    const TimingEvents ev = timing_events();
    if (ev.start && (e = cudaEventRecord(ev.start, stream)) != cudaSuccess) return e;
    if (pr.states_out) {
        // states only: one item per walk, the whole sequence, written to the
        // caller's [2][batch][H][kP][kN] states and [2][batch][H] decays
        TcParams q = p;
        q.seg_state = pr.states_out;
        q.seg_dec = pr.dec_out;
        q.nitems = 1;
        q.item_chunks = q.seg_chunks = p.nchunks;
        ssd_tc_kernel<true, false><<<dim3(d.heads, d.batch, 1), kThreads, kSmemBytes, stream>>>(
            tm_x_f, tm_x_r, tm_bc, q);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        count_launch();
        if (ev.stop) e = cudaEventRecord(ev.stop, stream);
        return e;
    }
    if (sp.nitems > 0) {
        TcParams q = p;
        q.seg_chunks = sp.item_chunks;   // one CTA per item
        ssd_tc_kernel<true, false><<<dim3(d.heads, d.batch, sp.nitems), kThreads, kSmemBytes, stream>>>(
            tm_x_f, tm_x_r, tm_bc, q);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        count_launch();
    }
    main_kernel<<<dim3(d.heads, d.batch, sp.nseg), kThreads, kSmemBytes, stream>>>(tm_x_f, tm_x_r, tm_bc,
                                                                                 p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    if (ev.stop) e = cudaEventRecord(ev.stop, stream);
    return e;
}

}  // namespace bimamba
