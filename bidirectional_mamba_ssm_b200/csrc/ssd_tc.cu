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
#include <type_traits>
#include <cuda.h>
#include <cudaTypedefs.h>

namespace bimamba {

namespace {

constexpr int kQ = 128;       // chunk length
constexpr int kP = 64;        // headdim of this kernel
constexpr int kN = 128;       // d_state of this kernel
constexpr int kHeads = 2;     // heads per CTA
constexpr int kPP = kHeads * kP;   // x channels per CTA (128)
constexpr int kGroupThreads = 256;        // each of the two compute groups (8 warps)
constexpr int kTmemWarps = 8;             // warps 0..7: the tensor-memory group
constexpr int kProducerWarp = 16;         // issues every MMA and TMA load
constexpr int kProducerTid = 32 * kProducerWarp;
constexpr int kHelperWarp = 17;           // dt copies, prefix sums, slot factors
constexpr int kPublisherWarp = 18;        // sets the meeting flags of stored rows
constexpr int kThreads = 2 * kGroupThreads + 96;
constexpr int kBC = 2 * kN;   // B and C channels
constexpr int kRawRows = kQ + 3;   // raw x rows per chunk: 128 slots + 3-token conv halo
constexpr uint32_t kTmemCols = 512;

// shared-memory map (bytes from a 1024-aligned base)
constexpr uint32_t kOffZlo = 0;        // 2 KB of zeros (block-diagonal B operand, below the X tiles)
constexpr uint32_t kOffC = 2048;       // C      [t][n]   2 x 16 KB (TMA, swizzled)
constexpr uint32_t kOffB = kOffC + 32768;   // B      [s][n]   2 x 16 KB (TMA, swizzled)
constexpr uint32_t kXbufBytes = 33792; // raw x [131][128] (TMA) -> X [s][p], 16 KB per head -> output rows
constexpr uint32_t kOffXbuf0 = kOffB + 32768;            // x buffer of even walk chunks
constexpr uint32_t kOffXbuf1 = kOffXbuf0 + kXbufBytes;   // odd walk chunks
constexpr uint32_t kOffXw = kOffXbuf1 + kXbufBytes;      // wX [s][p'] 2 x 16 KB
constexpr uint32_t kOffS = kOffXw + 32768;               // S^T bf16 [n][p'] 2 x 16 KB
constexpr uint32_t kOffZhi = kOffS + 32768;              // 2 KB of zeros (above the X tiles)
constexpr uint32_t kRawBytes = kRawRows * kPP * 2;       // 33536
constexpr uint32_t kOffCum = kOffZhi + 2048;     // f32[2][2][128] prefix sums of dt*A (chunk parity, head)
constexpr uint32_t kOffDt = kOffCum + 2048;      // f32[2][2][128] dt
constexpr uint32_t kOffFB = kOffDt + 2048;       // f32[2][2][128] exp(c_R - c_s) dt_s, R = block end
constexpr uint32_t kOffWgt = kOffFB + 2048;      // f32[2][2][128] exp(c_last - c_s) dt_s
constexpr uint32_t kOffF4 = kOffWgt + 2048;      // f32[2][2][128] exp(c_R4 - c_s) dt_s, R4 = s | 3
constexpr uint32_t kOffConvW = kOffF4 + 2048;    // float4[128] conv taps of x
constexpr uint32_t kOffConvB = kOffConvW + 16 * kPP;   // f32[128]
constexpr uint32_t kOffMbar = kOffConvB + 4 * kPP;     // u64 mbarriers (see the kernel)
constexpr uint32_t kOffTmem = kOffMbar + 192;    // u32 TMEM base
constexpr uint32_t kOffDtBuf = kOffTmem + 16;    // [2][128] bf16x2: dt of both heads, by cp.async
constexpr uint32_t kSmemUsed = kOffDtBuf + 2 * kQ * 4;
constexpr uint32_t kSmemBytes = kSmemUsed + 1024;   // + alignment slack
constexpr uint32_t kBCBytes = 4 * kQ * 64 * 2;      // four 128 x 64 bf16 boxes
static_assert(kOffC % 1024 == 0 && kOffB % 1024 == 0 && kOffXbuf0 % 1024 == 0, "tile alignment");
static_assert(kOffXbuf1 % 1024 == 0 && kOffXw % 1024 == 0 && kOffS % 1024 == 0, "tile alignment");
static_assert(kOffZhi % 1024 == 0, "tile alignment");
static_assert(kRawBytes <= kXbufBytes, "raw x tile must fit its buffer");
static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");

// TMEM columns.  Region A (0..127) holds G of a chunk, then, in place, its
// decay-masked M: the 16 columns of G for walk slots 16ks..16ks+15 become
// M_0 (8 columns of packed bf16 pairs) and M_1 (the next 8), K-step ks of
// the Yd product's A operand.  Region B (128..255) holds Yd, then Yo and the
// state are fixed.
constexpr uint32_t kColG = 0;
constexpr uint32_t kColYd = 128;   // + 64 * head
constexpr uint32_t kColYo = 256;   // + 64 * head
constexpr uint32_t kColS = 384;    // + 64 * head

constexpr long long kWaitCycles = 4000000000LL;  // ~2 s at 1.9 GHz

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
    // whole walks of tied directions: the partner CTA reads x chunk c and adds
    // to its y rows d = nchunks - 1 - 2k walk steps after this CTA (walk step
    // k); the first touches with 0 < d <= keep_dist stay in L2 (evict_last),
    // every other touch of x and y goes first (evict_first).  0: no hints.
    int keep_dist;
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

// Barrier over one compute group (named barrier `id`, 256 threads); the
// producer and helper warps never join it.
__device__ __forceinline__ void grp_sync(int id)
{
    asm volatile("bar.sync %0, 256;" :: "r"(id) : "memory");
}

__device__ __forceinline__ bool grp_sync_and(int id, bool pred)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.b32 p, %2, 0;\n\t"
        "bar.red.and.pred q, %1, 256, p;\n\t"
        "selp.b32 %0, 1, 0, q;\n\t}"
        : "=r"(r) : "r"(id), "r"((uint32_t)pred) : "memory");
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
    // every raw row of the thread's 8 steps (and the 3 before) requested at
    // once, kept as packed bf16
    uint4 rw[11];
#pragma unroll
    for (int i = 0; i < 11; ++i) {
        const int s = s_begin - 3 + i;
        if (s < s_end) {
            if (s >= 0) {
                rw[i] = *reinterpret_cast<const uint4 *>(xb + (size_t)(rev ? len - 1 - s : s) * ch);
            } else {
                float v[8];
                raw(s, v);
                rw[i] = pack8(v);
            }
        } else {
            rw[i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int s = s_begin + i;
        if (s >= s_end) break;
        float r0[8], r1[8], r2[8], r3[8], o[8];
        unpack8(rw[i], r0);
        unpack8(rw[i + 1], r1);
        unpack8(rw[i + 2], r2);
        unpack8(rw[i + 3], r3);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            float acc = bb[q];
            acc = fmaf(w0[q], r0[q], acc);
            acc = fmaf(w1[q], r1[q], acc);
            acc = fmaf(w2[q], r2[q], acc);
            acc = fmaf(w3[q], r3[q], acc);
            o[q] = tc::silu_tanh(acc);
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
//
// Warp roles (all communication through mbarriers; every wait is bounded):
//   warps 0..7   tensor-memory group: per chunk k, once its MMAs are done,
//                the output rows (Yd + exp(c) Yo, from TMEM) into the
//                chunk's x buffer (X is no longer needed); then M(k+1) in
//                place over G(k+1) and the state's chunk-start scaling with
//                its bf16 copy (the Yo operand).
//   warps 8..15  shared-memory group: per chunk k, wX(k+1) once the state
//                product of chunk k has read wX(k), and the in-place conv of
//                chunk k+2's raw rows.
//   warp 16      producer: every MMA, and the B/C tile loads.
//   warp 17      helper: dt copies, prefix sums and per-slot decay factors.
//   warp 18      publisher: per chunk k, the staged rows to y (the
//                forward/reverse meeting), then the raw rows of chunk k+2
//                into the freed x buffer.
// The two compute groups work on different chunks at the same time, and
// both overlap the tensor core.  In the state-only pass the shared-memory
// group only converts each chunk's x and hands it over; the tensor-memory
// group forms wX (double-buffered there in the unused bf16 state-copy tile,
// the B tiles in the unused C tile), releases the x buffer for the load of
// the chunk after next, and scales the state once the last product is done.
template <bool kStateOnly, bool kConcat>
__global__ void __launch_bounds__(kThreads, 1)
ssd_tc_kernel(const __grid_constant__ CUtensorMap tm_x_f, const __grid_constant__ CUtensorMap tm_x_r,
              const __grid_constant__ CUtensorMap tm_bc, const __grid_constant__ CUtensorMap tm_y,
              const TcParams p)
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
    // mbarriers (each completes once per walk chunk unless noted):
    const uint32_t mb_bc = sbase + kOffMbar;         // the chunk's B/C tiles landed
    const uint32_t mb_x0 = sbase + kOffMbar + 8;     // raw x landed in buffer 0 / 1 (+8)
    const uint32_t mb_g = sbase + kOffMbar + 24;     // G done
    const uint32_t mb_m = sbase + kOffMbar + 32;     // M ready (tensor-memory group)
    const uint32_t mb_e = sbase + kOffMbar + 40;     // the chunk's MMAs done
    const uint32_t mb_dt0 = sbase + kOffMbar + 48;   // an even / odd chunk's prefix sums and factors (+8)
    const uint32_t mb_free0 = sbase + kOffMbar + 64; // an even / odd chunk's factor buffers free (+8)
    const uint32_t mb_staged = sbase + kOffMbar + 80;   // the chunk's output rows staged
    const uint32_t mb_bcfree = sbase + kOffMbar + 88;   // the chunk's products that read B/C done
    const uint32_t mb_sdone = sbase + kOffMbar + 104;   // the chunk's state product done (wX read)
    const uint32_t mb_s = sbase + kOffMbar + 96;     // state, its bf16 copy and wX ready (one arrival per group)
    const uint32_t mb_yfree = sbase + kOffMbar + 112;   // Yd / Yo columns free for the chunk (last rows staged)
    const uint32_t mb_xr = sbase + kOffMbar + 120;      // (state-only pass) the chunk's X tile converted
    auto xbuf_off = [](int k) { return (k & 1) ? kOffXbuf1 : kOffXbuf0; };

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
        const void *tm = rev ? &tm_x_r : &tm_x_f;
        if (p.keep_dist == 0) {
            tc::tma_load_3d(sbase + xbuf_off(k), tm, hp * kPP, rev ? t0 : t0 - 3, b, mb);
        } else {
            const int d = nk - 1 - 2 * k;   // walk steps until the partner reads the chunk
            const uint64_t pol = (d > 0 && d <= p.keep_dist) ? tc::policy_evict_last() : tc::policy_evict_first();
            tc::tma_load_3d_hint(sbase + xbuf_off(k), tm, hp * kPP, rev ? t0 : t0 - 3, b, mb, pol);
        }
    };
    // chunk k's raw rows into L2 ahead of their load (the load of the chunk
    // after next is issued once the current one's buffer is free: by then its
    // rows come from L2, not HBM)
    auto prefetch_x = [&](int k) {
        int t0, cnt, s0;
        chunk_of(k, t0, cnt, s0);
        tc::tma_prefetch_l2_3d(rev ? &tm_x_r : &tm_x_f, hp * kPP, rev ? t0 : t0 - 3, b);
    };
    // B (and C) tiles of chunk k.  The state-only pass reads no C: there the
    // B tiles are double-buffered, odd chunks in the C tile on mbarrier mb_g
    // (no G there either)
    auto bbuf_off = [](int k) { return (kStateOnly && (k & 1)) ? kOffC : kOffB; };
    auto issue_bc = [&](int k) {
        int t0, cnt, s0;
        chunk_of(k, t0, cnt, s0);
        const int zc = dir * p.batch + b;
        const uint32_t mb = (kStateOnly && (k & 1)) ? mb_g : mb_bc;
        tc::mbar_expect_tx(mb, kStateOnly ? kBCBytes / 2 : kBCBytes);
        tc::tma_load_3d(sbase + bbuf_off(k), &tm_bc, 0, s0, zc, mb);
        tc::tma_load_3d(sbase + bbuf_off(k) + 16384, &tm_bc, 64, s0, zc, mb);
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
        // channel c = 4 cq + q of the pair stored at q * 32 + cq, so that
        // the 32 conv threads of a warp (channel quads cq) read 32
        // consecutive entries
        const int c = hp * kPP + tid;
        const int slot = (tid & 3) * 32 + (tid >> 2);
        const float4 w = *reinterpret_cast<const float4 *>(conv_w + (size_t)c * 4);
        convw[slot] = make_float4(0.5f * w.x, 0.5f * w.y, 0.5f * w.z, 0.5f * w.w);   // halved (see the conv)
        convb[slot] = conv_b ? 0.5f * conv_b[c] : 0.0f;
    }
    for (int i = tid; i < 2048 / 16; i += kThreads) {   // zero blocks of the block-diagonal Yd operand
        reinterpret_cast<uint4 *>(sm + kOffZlo)[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4 *>(sm + kOffZhi)[i] = make_uint4(0, 0, 0, 0);
    }
    if (warp == 0) tc::tmem_alloc(sbase + kOffTmem, kTmemCols);
    if (tid == kProducerTid) {
        tc::prefetch_tmap(rev ? &tm_x_r : &tm_x_f);
        tc::prefetch_tmap(&tm_bc);
        if (!kStateOnly) tc::prefetch_tmap(&tm_y);
        tc::mbar_init(mb_bc, 1);
        tc::mbar_init(mb_x0, 1);
        tc::mbar_init(mb_x0 + 8, 1);
        tc::mbar_init(mb_g, 1);
        tc::mbar_init(mb_m, 1);
        // one arrival from each compute group (the state-only pass: from the
        // tensor-memory group, which forms w o X there too)
        tc::mbar_init(mb_s, kStateOnly ? 1 : 2);
        tc::mbar_init(mb_xr, 1);
        tc::mbar_init(mb_e, 1);
        tc::mbar_init(mb_dt0, 32);       // every helper lane arrives after its part of a scan
        tc::mbar_init(mb_dt0 + 8, 32);
        tc::mbar_init(mb_free0, 2);      // both compute groups done with the factors
        tc::mbar_init(mb_free0 + 8, 2);
        tc::mbar_init(mb_staged, 1);
        tc::mbar_init(mb_bcfree, 1);
        tc::mbar_init(mb_sdone, 1);
        tc::mbar_init(mb_yfree, 1);
        issue_x(0);
        if (nk > 1) issue_x(1);
        if (!kStateOnly && nk > 2) prefetch_x(2);
        issue_bc(0);
        if (kStateOnly && nk > 1) issue_bc(1);
    }
    if (warp == kHelperWarp) {
        load_dt_async(0);
        if (nk > 1) load_dt_async(1);
    }
    tc::fence_proxy_async();   // the zero blocks, for the tensor core
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + kOffTmem);

    // wX = w_s * X for walk chunk k (X tile in x buffer k % 2): thread
    // tt (slot j, head gh), the head's 64 channels
    auto wxbuf_off = [](int k) { return (kStateOnly && (k & 1)) ? kOffS : kOffXw; };
    auto weight_chunk = [&](int k, int tt) {
        // in bf16 pairs: w_s rounded to bf16, each product rounded once
        // (the state-only pass alternates two wX tiles)
        const uint8_t *xt = sm + xbuf_off(k);
        uint8_t *wx = sm + wxbuf_off(k);
        const int j = tt & 127, gh = tt >> 7;
        const __nv_bfloat162 w2 = __float2bfloat162_rn(wgt[((k & 1) * kHeads + gh) * kQ + j]);
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {
            const uint32_t off = gh * 16384 + tc::sw128(j, pc);
            uint4 v = *reinterpret_cast<const uint4 *>(xt + off);
            __nv_bfloat162 *h2 = reinterpret_cast<__nv_bfloat162 *>(&v);
#pragma unroll
            for (int q = 0; q < 4; ++q) h2[q] = __hmul2(h2[q], w2);
            *reinterpret_cast<uint4 *>(wx + off) = v;
        }
    };

    if (warp == kProducerWarp) {
        // ================= producer: every MMA and every TMA load (lane 0)
        const uint64_t dC = tc::smem_desc(sbase + kOffC, 16, 1024);       // K-major A (G, Yo)
        const uint64_t dB = tc::smem_desc(sbase + kOffB, 16, 1024);       // K-major B (G)
        const uint64_t dBmn = tc::smem_desc(sbase + kOffB, 16384, 1024);  // MN-major A (state)
        const uint64_t dS = tc::smem_desc(sbase + kOffS, 16384, 1024);    // MN-major B (Yo)
        const uint64_t dXw = tc::smem_desc(sbase + kOffXw, 16384, 1024);  // MN-major B (state)
        constexpr uint32_t idG = tc::idesc_bf16(128, 128, 0, 0);
        constexpr uint32_t idY = tc::idesc_bf16(128, 128, 0, 1);
        constexpr uint32_t idS = tc::idesc_bf16(128, 128, 1, 1);
        auto issue_g = [&]() {
#pragma unroll 1
            for (int ks = 0; ks < kN / 16; ++ks) {
                const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                tc::mma_bf16(tmem + kColG, tc::desc_add(dC, koff), tc::desc_add(dB, koff), idG, ks > 0);
            }
            tc::mma_commit(mb_g);
        };
        bool pok = true;
        if (lane == 0) {
            if (!kStateOnly) {
                pok = tc::mbar_wait_bounded(mb_bc, 0, kWaitCycles);
                if (pok) {
                    tc::fence_after_sync();
                    issue_g();
                }
            }
            for (int k = 0; k < nk && pok; ++k) {
                // the state scaled for this chunk, its bf16 copy and wX
                pok = tc::mbar_wait_bounded(mb_s, k & 1, kWaitCycles);
                if (pok && kStateOnly)
                    pok = tc::mbar_wait_bounded((k & 1) ? mb_g : mb_bc, (k >> 1) & 1, kWaitCycles);
                if (!pok) break;
                tc::fence_after_sync();
                // the state product first: the next chunk's state scaling waits for it
                const uint64_t dBk = kStateOnly ? tc::smem_desc(sbase + bbuf_off(k), 16384, 1024) : dBmn;
                const uint64_t dXwk = kStateOnly ? tc::smem_desc(sbase + wxbuf_off(k), 16384, 1024) : dXw;
#pragma unroll 1
                for (int ks = 0; ks < kQ / 16; ++ks)
                    tc::mma_bf16(tmem + kColS, tc::desc_add(dBk, ks * 2048), tc::desc_add(dXwk, ks * 2048),
                                 idS, 1);
                if constexpr (!kStateOnly) {
                    tc::mma_commit(mb_sdone);   // wX may be rewritten once it completes
                    // Yo = C S_in^T (both heads), once the last chunk's rows are out of TMEM
                    pok = tc::mbar_wait_bounded(mb_yfree, k & 1, kWaitCycles);
                    if (!pok) break;
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int ks = 0; ks < kN / 16; ++ks) {
                        const uint32_t koff = (ks >> 2) * 16384 + (ks & 3) * 32;
                        tc::mma_bf16(tmem + kColYo, tc::desc_add(dC, koff), tc::desc_add(dS, ks * 2048), idY,
                                     ks > 0);
                    }
                    // the B/C tiles are free once the state product and Yo are
                    // done: the next chunk's tiles load while Yd runs
                    tc::mma_commit(mb_bcfree);
                    // M, built while the two products above run
                    pok = tc::mbar_wait_bounded(mb_m, k & 1, kWaitCycles);
                    if (!pok) break;
                    tc::fence_after_sync();
                    // Yd = [M_0 | M_1] . [[X_0, 0], [0, X_1]]: one N = 128 product over
                    // K = 256.  K-steps 0..7 take X_0's rows as N block 0 and the
                    // zeros above the tiles as N block 1 (leading offset = the
                    // distance to them); K-steps 8..15 the zeros below as N block 0
                    // and X_1's rows as N block 1.
                    const uint32_t xb = sbase + xbuf_off(k);
                    const uint64_t d0 = tc::smem_desc(xb, sbase + kOffZhi - xb, 1024);
                    const uint64_t d1 = tc::smem_desc(sbase + kOffZlo, xb + 16384 - (sbase + kOffZlo), 1024);
                    constexpr uint64_t kStep0 = 128ull - (128ull << 16);   // start += 2 KB, offset -= 2 KB
                    constexpr uint64_t kStep1 = 128ull << 16;              // offset += 2 KB
#pragma unroll 1
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16_tmemA(tmem + kColYd, tmem + kColG + 16 * ks, d0 + ks * kStep0, idY, ks > 0);
#pragma unroll 1
                    for (int ks = 0; ks < 8; ++ks)
                        tc::mma_bf16_tmemA(tmem + kColYd, tmem + kColG + 16 * ks + 8, d1 + ks * kStep1, idY, 1);
                }
                tc::mma_commit(mb_e);
                if (k + 1 >= nk) break;
                if constexpr (!kStateOnly) {
                    pok = tc::mbar_wait_bounded(mb_bcfree, k & 1, kWaitCycles);
                    if (!pok) break;
                    issue_bc(k + 1);
                }
                // once all of them complete: this chunk's x buffer and TMEM
                // region A are free
                pok = tc::mbar_wait_bounded(mb_e, k & 1, kWaitCycles);
                if (!pok) break;
                if constexpr (kStateOnly) {
                    // B buffer k % 2 is free (the tensor-memory group issues the x loads)
                    if (k + 2 < nk) issue_bc(k + 2);
                }
                if constexpr (!kStateOnly) {
                    pok = tc::mbar_wait_bounded(mb_bc, (k + 1) & 1, kWaitCycles);
                    if (!pok) break;
                    tc::fence_after_sync();
                    issue_g();
                }
            }
            if (!pok) record_error(p.status, kStatusTimeout);
        }
        __syncwarp();
    } else if (warp == kPublisherWarp) {
        // ================= publisher: chunk k's output rows, staged by the
        // tensor-memory group in x buffer k % 2 (free once the chunk's MMAs
        // are done), to y, and the forward + reverse sum.  The two CTAs of a
        // (sequence, head pair) meet per token chunk: the first to arrive
        // stores its rows, the second adds its own to them (bf16 reductions
        // at L2) once the first has set the chunk's ready flag.  Then x
        // buffer k % 2 takes chunk k+2's raw rows (TMA, issued here).
        if constexpr (!kStateOnly) {
            bool qok = true;
            const int col0 = (kConcat ? dir * H * kP : 0) + hp * kPP;   // the head pair's first y column
            for (int k = 0; k < nk && qok && lane == 0; ++k) {
                int t0, cnt, s0;
                const int c = chunk_of(k, t0, cnt, s0);
                int *fl = p.flags + (((size_t)b * HP + hp) * p.nchunks + c) * 2;
                const int arrival = kConcat ? 0 : atomicAdd(fl, 1);
                qok = tc::mbar_wait_bounded(mb_staged, k & 1, kWaitCycles);
                if (!qok) break;
                const bool first = arrival == 0;
                const uint32_t stg = sbase + xbuf_off(k);
                // (whole walks) the partner adds to these rows |d| walk steps from now
                const int d = nk - 1 - 2 * k;
                const bool hint = p.keep_dist > 0;
                const uint64_t pol = (first && abs(d) <= p.keep_dist) ? tc::policy_evict_last()
                                                                      : tc::policy_evict_first();
                if (first) {
                    if (hint) {
                        tc::tma_store_3d_hint(&tm_y, stg, col0, t0, b, pol);
                        tc::tma_store_3d_hint(&tm_y, stg + 16384, col0 + kP, t0, b, pol);
                    } else {
                        tc::tma_store_3d(&tm_y, stg, col0, t0, b);
                        tc::tma_store_3d(&tm_y, stg + 16384, col0 + kP, t0, b);
                    }
                } else {
                    // the partner CTA arrived first; wait (bounded) until its
                    // rows are visible, then add this CTA's to them at L2.  A
                    // wait that gave up stops the walk here: the partner's rows
                    // are not added to, and the meeting counters are left as
                    // they are (the caller zero-fills the workspace again
                    // after a timeout).
                    bool ready;
                    const long long w0 = clock64();
                    while (!(ready = ld_acquire(fl + 1) != 0)) {
                        if (clock64() - w0 > kWaitCycles) break;
                    }
                    qok = ready;
                    if (!qok) break;
                    tc::fence_proxy_async_global();   // the acquire before the reductions
                    if (hint) {
                        tc::tma_reduce_add_3d_hint(&tm_y, stg, col0, t0, b, pol);
                        tc::tma_reduce_add_3d_hint(&tm_y, stg + 16384, col0 + kP, t0, b, pol);
                    } else {
                        tc::tma_reduce_add_3d(&tm_y, stg, col0, t0, b);
                        tc::tma_reduce_add_3d(&tm_y, stg + 16384, col0 + kP, t0, b);
                    }
                }
                tc::bulk_commit();
                tc::bulk_wait_read0();   // the staged rows have been read
                if (k + 2 < nk) issue_x(k + 2);
                if (k + 3 < nk) prefetch_x(k + 3);
                if (!kConcat) {
                    if (first) {
                        // publish the rows to the partner once written
                        tc::bulk_wait0();
                        tc::fence_proxy_async_global();
                        st_release(fl + 1, 1);
                    } else {
                        fl[0] = 0;   // leave the workspace zeroed for the next call
                        fl[1] = 0;
                    }
                }
            }
            if (lane == 0) tc::bulk_wait0();
            if (lane == 0 && !qok) record_error(p.status, kStatusTimeout);
        }
        __syncwarp();
    } else if (warp == kHelperWarp) {
        // ================= helper: dt copies, prefix sums and slot factors
        // of each chunk, up to two chunks ahead (the copies of chunks 0 and 1
        // were issued before the set-up barrier)
        bool hok = true;
        for (int j = 0; j < nk; ++j) {
            if (j >= 2) {
                // buffer j % 2 last held chunk j-2: wait until both groups are done with it
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
    } else if (warp < kTmemWarps) {
        // ================= tensor-memory group (warps 0..7) ================
        // thread (row, h): TMEM lane `row` (token slot t, or state row n), head h
        const int row = tid & 127;
        const int h = tid >> 7;
        const int quad = warp & 3;
        const uint32_t lane_base = static_cast<uint32_t>(32 * quad) << 16;
        const int head_g = hp * kHeads + h;
        auto a_wait = [&](uint32_t mb, uint32_t parity) -> bool {
            bool w = true;
            if (tid == 0) w = tc::mbar_wait_bounded(mb, parity, kWaitCycles);
            return grp_sync_and(1, w);
        };
        // ---- the state entering the walk, S^T[n = row][p] of head h ->
        // TMEM columns kColS + 64 h: the caller's initial state (forward) or
        // zero, carried through the shards before this one (sequence shards)
        // and the items before this segment: S <- 2^dec_i S + S_i.
        {
            const size_t sidx = ((size_t)b * H + head_g) * kP * kN;
            const bool use_init = !kStateOnly && !rev && p.init;
            const int n_sh = (kStateOnly || !p.shard_states) ? 0 : (rev ? p.nranks - 1 - p.rank : p.rank);
            const int n_in = (kStateOnly || p.item_chunks == 0) ? 0 : k0 / p.item_chunks;
#pragma unroll 1
            for (int q16 = 0; q16 < 4; ++q16) {
                float v[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    v[i] = use_init ? __ldg(p.init + sidx + (size_t)(16 * q16 + i) * kN + row) : 0.0f;
                for (int it = 0; it < n_sh; ++it) {
                    const int q = rev ? p.nranks - 1 - it : it;
                    const size_t e = (((size_t)q * 2 + dir) * p.batch + b) * H + head_g;
                    const float *si = p.shard_states + e * kP * kN;
                    const float a = tc::exp2_approx(p.shard_dec[e]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = fmaf(v[i], a, si[(size_t)(16 * q16 + i) * kN + row]);
                }
                for (int it = 0; it < n_in; ++it) {
                    const float *si = p.seg_state + ((item_row + it) * kHeads + h) * kP * kN;
                    const float a = tc::exp2_approx(p.seg_dec[(item_row + it) * kHeads + h]);
#pragma unroll
                    for (int i = 0; i < 16; ++i) v[i] = fmaf(v[i], a, si[(size_t)(16 * q16 + i) * kN + row]);
                }
                uint32_t r[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(v[i]);
                tc::tmem_st16(tmem + lane_base + kColS + 64 * h + 16 * q16, r);
            }
        }
        // D of both heads of the pair (M's diagonal; a thread builds both)
        const float *Dpair = (rev ? p.D[1] : p.D[0]) + hp * kHeads;
        const float D0 = kStateOnly ? 0.0f : Dpair[0], D1 = kStateOnly ? 0.0f : Dpair[1];
        float dec = 0.0f;   // state-only: the item's total decay (log2 units)

        // M(k) in place over G(k) (region A): thread (t = row, h) owns the
        // walk slots of 32-slot blocks 2h, 2h+1 for both heads.  The 16 G
        // columns of slots 16ks..16ks+15 become [M_0 ks | M_1 ks] (8 + 8
        // columns of packed bf16 pairs), so no other thread reads them.  One
        // TMEM load per block; the stores are not waited for here (the caller
        // waits once before publishing M).
        auto build_m = [&](int k) {
            const int row = tc::no_hoist(tid & 127);   // (see no_hoist)
            const int par = k & 1;
            // 16-slot units U = 2 jb + u (K-steps of Yd) of this quarter's rows:
            // units past the quarter's own block are all zero (s > t); of the
            // others, warp h takes factorised units h*quad .. h*quad+quad-1 and
            // diagonal unit 2 quad + h, so both warps of a quarter carry the same
            // load
            {
                uint32_t z[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll 1
                for (int U = 2 * quad + 2 + h; U < 8; U += 2) tc::tmem_st16_nw(tmem + lane_base + kColG + 16 * U, z);
            }
#pragma unroll 1
            for (int iu = 0; iu <= quad; ++iu) {
                const int U = iu < quad ? h * quad + iu : 2 * quad + h;
                const int jb = U >> 1, u = U & 1;   // 32-slot block of s, half of it
                const uint32_t col = tmem + lane_base + kColG + 32 * jb;
                {
                    uint32_t gu[16];
                    tc::tmem_ld16_nw(col + 16 * u, gu);
                    tc::tmem_wait_ld16(gu);
                    const int s0u = 32 * jb + 16 * u;   // first slot of the unit
#pragma unroll 1
                    for (int hd = 0; hd < kHeads; ++hd) {
                        const float *cm = cum + (par * kHeads + hd) * kQ;
                        const float ct = cm[row];
                        uint32_t out[8];            // head hd's 8 packed pairs
                        if (jb < quad) {
                            // whole block below the diagonal: factorised decay
                            const float2 *fbh = reinterpret_cast<const float2 *>(fB + (par * kHeads + hd) * kQ + s0u);
                            const float et = tc::exp2_approx(ct - cm[32 * jb + 31]);
                            const float2 et2 = make_float2(et, et);
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const float2 g2 = make_float2(__uint_as_float(gu[2 * i]),
                                                              __uint_as_float(gu[2 * i + 1]));
                                const float2 m = tc::mul2(tc::mul2(g2, et2), fbh[i]);
                                out[i] = tc::pack_bf16x2(m.x, m.y);
                            }
                        } else {
                            // diagonal block, D on the diagonal; slot s0u + i
                            // against t's offset r in the unit
                            const int r = (row & 31) - 16 * u;
                            const float Dh = hd ? D1 : D0;
                            if (cm[32 * jb] - cm[32 * jb + 31] <= 60.0f) {   // warp-uniform (head, block)
                                // 4-slot sub-blocks: exp(c_t - c_s) = exp(c_t - c_R4)
                                // exp(c_R4 - c_s), R4 = s | 3.  With the block's whole
                                // decay at most 2^60 neither factor overflows; for s <= t
                                // the product is the decay itself
                                const float *f4h = f4 + (par * kHeads + hd) * kQ + s0u;
#pragma unroll
                                for (int q4 = 0; q4 < 4; ++q4) {
                                    const float rf = tc::exp2_approx(ct - cm[s0u + 4 * q4 + 3]);
                                    float v[4];
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int i = 4 * q4 + e;
                                        const float x = fmaf(__uint_as_float(gu[i]) * rf, f4h[i],
                                                             (i == r) ? Dh : 0.0f);
                                        v[e] = (i <= r) ? x : 0.0f;
                                    }
                                    out[2 * q4] = tc::pack_bf16x2(v[0], v[1]);
                                    out[2 * q4 + 1] = tc::pack_bf16x2(v[2], v[3]);
                                }
                            } else {
                                // steep decays: one exponential per element, each <= 1
                                const float *dh_ = dts + (par * kHeads + hd) * kQ + s0u;
#pragma unroll
                                for (int i2 = 0; i2 < 8; ++i2) {
                                    float v[2];
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        const int i = 2 * i2 + e;
                                        const float ex = tc::exp2_approx(fminf(ct - cm[s0u + i], 0.0f));
                                        const float x = fmaf(__uint_as_float(gu[i]) * ex, dh_[i],
                                                             (i == r) ? Dh : 0.0f);
                                        v[e] = (i <= r) ? x : 0.0f;
                                    }
                                    out[i2] = tc::pack_bf16x2(v[0], v[1]);
                                }
                            }
                        }
                        tc::tmem_st8_nw(col + 16 * u + 8 * hd, out);
                    }
                }
            }
        };
        // the state at chunk k's start: bf16 copy of S_in (the Yo operand),
        // then S <- exp(c_last) S in place (stores not waited for here)
        auto scale_state = [&](int k) {
            const int row = tc::no_hoist(tid & 127);   // (see no_hoist)
            const float cl = cum[((k & 1) * kHeads + h) * kQ + kQ - 1];
            const float a_last = tc::exp2_approx(cl);
            const float2 a2 = make_float2(a_last, a_last);
            if constexpr (kStateOnly) dec += cl;
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                uint32_t sr[32];
                const uint32_t col = tmem + lane_base + kColS + 64 * h + 32 * half;
                tc::tmem_ld32_nw(col, sr);
                tc::tmem_wait_ld(sr);
                if constexpr (!kStateOnly) {
#pragma unroll
                    for (int pc = 0; pc < 4; ++pc) {
                        uint4 w;
                        w.x = tc::pack_bf16x2(__uint_as_float(sr[8 * pc]), __uint_as_float(sr[8 * pc + 1]));
                        w.y = tc::pack_bf16x2(__uint_as_float(sr[8 * pc + 2]), __uint_as_float(sr[8 * pc + 3]));
                        w.z = tc::pack_bf16x2(__uint_as_float(sr[8 * pc + 4]), __uint_as_float(sr[8 * pc + 5]));
                        w.w = tc::pack_bf16x2(__uint_as_float(sr[8 * pc + 6]), __uint_as_float(sr[8 * pc + 7]));
                        *reinterpret_cast<uint4 *>(sm + kOffS + h * 16384 + tc::sw128(row, 4 * half + pc)) = w;
                    }
                }
#pragma unroll
                for (int half16 = 0; half16 < 2; ++half16) {
                    uint32_t r[16];
#pragma unroll
                    for (int i = 0; i < 16; i += 2) {
                        const float2 v = tc::mul2(make_float2(__uint_as_float(sr[16 * half16 + i]),
                                                              __uint_as_float(sr[16 * half16 + i + 1])), a2);
                        r[i] = __float_as_uint(v.x);
                        r[i + 1] = __float_as_uint(v.y);
                    }
                    tc::tmem_st16_nw(col + 16 * half16, r);
                }
            }
        };
        // chunk k's output rows, y = Yd + exp(c_t) Yo, into the chunk's x
        // buffer (free once its MMAs are done) as two TMA store boxes, one
        // per head: [token row of the chunk][64 channels], 128-byte rows,
        // 16-byte piece j of row q at j ^ (q & 7).  The reverse stream's
        // walk slot r is token row cnt - 1 - r; slots past the chunk end are
        // not written (the box rows past the sequence end are not stored).
        auto stage_rows = [&](int k) {
            const int row = tc::no_hoist(tid & 127);   // (see no_hoist)
            int t0, cnt, s0;
            chunk_of(k, t0, cnt, s0);
            const int q = rev ? cnt - 1 - row : row;   // token row in the box
            uint8_t *box = sm + xbuf_off(k) + h * 16384 + q * 128;
            const float et = tc::exp2_approx(cum[((k & 1) * kHeads + h) * kQ + row]);
            const float2 et2 = make_float2(et, et);
#pragma unroll 1
            for (int qtr = 0; qtr < 4; ++qtr) {
                uint32_t yy[32];   // [0, 16): Yd, [16, 32): Yo
                tc::tmem_ld16_nw(tmem + lane_base + kColYd + 64 * h + 16 * qtr, yy);
                tc::tmem_ld16_nw(tmem + lane_base + kColYo + 64 * h + 16 * qtr, yy + 16);
                tc::tmem_wait_ld(yy);
#pragma unroll
                for (int pc = 0; pc < 2; ++pc) {
                    float v[8];
#pragma unroll
                    for (int i = 0; i < 8; i += 2) {
                        const int e = 8 * pc + i;
                        const float2 y2 = tc::fma2(et2, make_float2(__uint_as_float(yy[16 + e]), __uint_as_float(yy[17 + e])),
                                                   make_float2(__uint_as_float(yy[e]), __uint_as_float(yy[e + 1])));
                        v[i] = y2.x;
                        v[i + 1] = y2.y;
                    }
                    const int piece = 2 * qtr + pc;
                    if (q >= 0) *reinterpret_cast<uint4 *>(box + ((piece ^ (q & 7)) << 4)) = pack8(v);
                }
            }
        };
        // publish this group's part of a chunk's MMA operands on mbarrier mb
        auto publish = [&](uint32_t mb, bool smem_operands) {
            tc::tmem_wait_st();
            if (smem_operands) tc::fence_proxy_async();   // the bf16 state copy, for the tensor core
            tc::fence_before_sync();
            grp_sync(1);
            if (tid == 0) tc::mbar_arrive(mb);
        };

        // Per chunk k: the state at its start (the operands of the state
        // product and Yo) first, then M(k) (the operand of Yd), so that the
        // producer issues the first two products while M is being built.
        // Per walk chunk j: once chunk j-1's MMAs are done, its output rows;
        // then the state at chunk j's start (the operands of the state
        // product and Yo) first, and M(j) (the operand of Yd), so that the
        // producer issues the first two products while M is being built.
        // (Every phase has one call site.)
        bool ok = true;
        if constexpr (kStateOnly) {
            // per chunk, once the other group has converted its x: the state
            // scaling and w o X (so that the conv group never waits on the
            // products)
            for (int j = 0; j < nk && ok; ++j) {
                // w o X of chunk j into wX tile j % 2 (the product of chunk
                // j-2 read it: waited for in the last iteration)
                ok = a_wait(mb_xr, j & 1);
                if (ok) ok = a_wait(mb_dt0 + 8 * (j & 1), (j >> 1) & 1);
                if (!ok) break;
                tc::fence_after_sync();
                weight_chunk(j, tid);
                grp_sync(1);   // x buffer j % 2 read: the load of chunk j+2 may overwrite it
                if (tid == 0) {
                    tc::mbar_arrive(mb_free0 + 8 * (j & 1));
                    if (j + 2 < nk) issue_x(j + 2);
                }
                if (j >= 1) ok = a_wait(mb_e, (j - 1) & 1);   // the last product has updated the state
                if (!ok) break;
                tc::fence_after_sync();
                scale_state(j);
                publish(mb_s, true);
            }
            if (ok) {
                ok = a_wait(mb_e, (nk - 1) & 1);   // the last chunk's product
                tc::fence_after_sync();
            }
        } else {
            for (int j = 0; j <= nk && ok; ++j) {
                if (j >= 1) {
                    ok = a_wait(mb_e, (j - 1) & 1);   // chunk j-1's MMAs done
                    if (!ok) break;
                    tc::fence_after_sync();
                }
                if (j < nk) {
                    // the state for chunk j first: its product runs while the rows
                    // of chunk j-1 are read out
                    ok = a_wait(mb_dt0 + 8 * (j & 1), (j >> 1) & 1);   // chunk j's prefix sums and factors
                    if (!ok) break;
                    tc::fence_after_sync();
                    scale_state(j);
                    publish(mb_s, !kStateOnly);
                }
                if (j >= 1) {
                    if constexpr (!kStateOnly) {
                        stage_rows(j - 1);
                        tc::fence_proxy_async();   // the staged rows, for the publisher's TMA stores
                        tc::fence_before_sync();   // TMEM reads done before the next chunk's products
                        grp_sync(1);
                        if (tid == 0) {
                            tc::mbar_arrive(mb_staged);
                            if (j < nk) tc::mbar_arrive(mb_yfree);
                        }
                    }
                    if (tid == 0) tc::mbar_arrive(mb_free0 + 8 * ((j - 1) & 1));
                    if (j >= nk) break;
                } else if (!kStateOnly && tid == 0) {
                    tc::mbar_arrive(mb_yfree);   // nothing staged before chunk 0
                }
                if constexpr (!kStateOnly) {
                    ok = a_wait(mb_g, j & 1);
                    if (!ok) break;
                    tc::fence_after_sync();
                    build_m(j);
                    publish(mb_m, false);
                }
            }
        }
        if (ok) {
            // the last chunk's MMAs are done (waited above)
            if constexpr (kStateOnly) {
                // the item's end state and total decay
                const size_t item = item_row + blockIdx.z;
                float *so = p.seg_state + (item * kHeads + h) * kP * kN;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float sv[32];
                    tc::tmem_ld32(tmem + lane_base + kColS + 64 * h + 32 * half, sv);
#pragma unroll
                    for (int i = 0; i < 32; ++i) so[(size_t)(32 * half + i) * kN + row] = sv[i];
                }
                if (row == 0) p.seg_dec[item * kHeads + h] = dec;
            } else if (!rev && p.fin && k0 + nk == p.nchunks) {
                const size_t sidx = ((size_t)b * H + head_g) * kP * kN;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    float sv[32];
                    tc::tmem_ld32(tmem + lane_base + kColS + 64 * h + 32 * half, sv);
#pragma unroll
                    for (int i = 0; i < 32; ++i) p.fin[sidx + (size_t)(32 * half + i) * kN + row] = sv[i];
                }
            }
        }
        if (!ok && tid == 0) record_error(p.status, kStatusTimeout);
    } else {
        // ================= shared-memory group (warps 8..15) ===============
        const int tb = tid - kGroupThreads;   // 0..255
        auto b_wait = [&](uint32_t mb, uint32_t parity) -> bool {
            bool w = true;
            if (tb == 0) w = tc::mbar_wait_bounded(mb, parity, kWaitCycles);
            return grp_sync_and(2, w);
        };
        // conv+SiLU of both heads' x for walk chunk k, in place: the raw
        // rows in x buffer k % 2 become the swizzled X tile of the chunk.
        // Thread: channel quad cq (channels 4cq .. 4cq+3, head cq >> 4) x 16
        // walk slots 16sg .. 16sg+15, in packed fp32 pairs.  The raw row of
        // slot s's tap j is s + j forward (the box starts 3 tokens early)
        // and cnt + 2 - s - j reverse (the mirror image); the direction is a
        // compile-time constant of each instance.  Every thread reads its
        // raw rows before the group barrier and writes after it.  The taps
        // and bias are stored halved: SiLU(a) = h + h tanh(h) with h = a / 2.
        auto conv_impl = [&](auto rev_c, int k) {
            constexpr bool kR = decltype(rev_c)::value;
            int t0, cnt, s0;
            chunk_of(k, t0, cnt, s0);
            uint8_t *buf = sm + xbuf_off(k);
            const int cq = tb & 31, sg = tb >> 5;
            const int j0 = 16 * sg;
            // reverse rows below 0 (slots past a short chunk's end) read other
            // shared memory of this CTA; those slots are written as zeros
            const uint8_t *src = buf + (kR ? cnt + 2 - j0 : j0) * (kPP * 2) + 8 * cq;
            uint2 rr[19];
#pragma unroll
            for (int i = 0; i < 19; ++i)
                rr[i] = *reinterpret_cast<const uint2 *>(src + (kR ? -i : i) * (kPP * 2));
            grp_sync(2);
            uint8_t *dst = buf + (cq >> 4) * 16384 + j0 * 128 + 8 * (cq & 1);
            const uint32_t pbase = static_cast<uint32_t>((cq & 15) >> 1) << 4;   // piece, before the swizzle
            const bool full = j0 + 16 <= cnt;
            auto up = [](uint32_t r) {
                return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&r));
            };
            if (has_conv) {
                float4 wq[4];
                float bq[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    wq[q] = convw[q * 32 + cq];
                    bq[q] = convb[q * 32 + cq];
                }
                // channel pairs (0, 1) and (2, 3) of the quad, per tap
                const float2 wa0 = make_float2(wq[0].x, wq[1].x), wa1 = make_float2(wq[0].y, wq[1].y);
                const float2 wa2 = make_float2(wq[0].z, wq[1].z), wa3 = make_float2(wq[0].w, wq[1].w);
                const float2 wb0 = make_float2(wq[2].x, wq[3].x), wb1 = make_float2(wq[2].y, wq[3].y);
                const float2 wb2 = make_float2(wq[2].z, wq[3].z), wb3 = make_float2(wq[2].w, wq[3].w);
                const float2 ba = make_float2(bq[0], bq[1]), bb = make_float2(bq[2], bq[3]);
                float2 a0 = up(rr[0].x), a1 = up(rr[1].x), a2 = up(rr[2].x);
                float2 b0 = up(rr[0].y), b1 = up(rr[1].y), b2 = up(rr[2].y);
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 a3 = up(rr[i + 3].x), b3 = up(rr[i + 3].y);
                    float2 ha = tc::fma2(wa0, a0, ba);
                    float2 hb = tc::fma2(wb0, b0, bb);
                    ha = tc::fma2(wa1, a1, ha);
                    hb = tc::fma2(wb1, b1, hb);
                    ha = tc::fma2(wa2, a2, ha);
                    hb = tc::fma2(wb2, b2, hb);
                    ha = tc::fma2(wa3, a3, ha);
                    hb = tc::fma2(wb3, b3, hb);
                    float t[4];
                    asm("tanh.approx.f32 %0, %1;" : "=f"(t[0]) : "f"(ha.x));
                    asm("tanh.approx.f32 %0, %1;" : "=f"(t[1]) : "f"(ha.y));
                    asm("tanh.approx.f32 %0, %1;" : "=f"(t[2]) : "f"(hb.x));
                    asm("tanh.approx.f32 %0, %1;" : "=f"(t[3]) : "f"(hb.y));
                    const float2 oa = tc::fma2(ha, make_float2(t[0], t[1]), ha);
                    const float2 ob = tc::fma2(hb, make_float2(t[2], t[3]), hb);
                    uint2 pk = make_uint2(tc::pack_bf16x2(oa.x, oa.y), tc::pack_bf16x2(ob.x, ob.y));
                    if (!full && j0 + i >= cnt) pk = make_uint2(0u, 0u);
                    *reinterpret_cast<uint2 *>(dst + i * 128 + (pbase ^ ((i & 7) << 4))) = pk;
                    a0 = a1; a1 = a2; a2 = a3;
                    b0 = b1; b1 = b2; b2 = b3;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    uint2 pk = rr[i + 3];
                    if (!full && j0 + i >= cnt) pk = make_uint2(0u, 0u);
                    *reinterpret_cast<uint2 *>(dst + i * 128 + (pbase ^ ((i & 7) << 4))) = pk;
                }
            }
        };
        auto conv_chunk = [&](int k) {
            if (rev)
                conv_impl(std::true_type{}, k);
            else
                conv_impl(std::false_type{}, k);
        };
        // sequence shards: the reverse stream's conv reads the 3 tokens
        // after the shard (L .. L+2) from the head.  Raw row i of a reverse
        // chunk buffer is token t0 + i, so they land in the walk's first
        // chunk and, when that chunk holds fewer than 3 tokens, also in the
        // second (whose TMA box ran past the shard end and read zeros).
        auto head_rows = [&](int k) {
            if (!rev || !p.head) return;
            int t0, cnt, s0;
            chunk_of(k, t0, cnt, s0);
            if (L - t0 >= kRawRows) return;
            const uint32_t buf = xbuf_off(k);
            for (int e = tb; e < 3 * (kPP / 8); e += kGroupThreads) {
                const int r = e / (kPP / 8), g = e % (kPP / 8);
                const int row = L - t0 + r;
                if (row < kRawRows)
                    *reinterpret_cast<uint4 *>(sm + buf + row * (kPP * 2) + g * 16) =
                        *reinterpret_cast<const uint4 *>(p.head + ((size_t)b * 4 + r) * ch +
                                                         hp * kPP + 8 * g);
            }
            grp_sync(2);
        };

        // Per walk chunk j: the conv of its raw rows (x buffer j % 2), then
        // wX(j) = w o X(j) once the state product of chunk j-1 has read
        // wX(j-1).  (Every phase has one call site: the kernel's code stays
        // small enough for the instruction caches.)
        bool ok = true;
        if constexpr (kStateOnly) {
            // per chunk: its raw rows (and halos) converted in place, handed to
            // the tensor-memory group, which forms w o X
            for (int j = 0; j < nk && ok; ++j) {
                ok = b_wait(mb_x0 + 8 * (j & 1), (j >> 1) & 1);
                if (!ok) break;
                if (j == 0 && !rev && p.tail && k0 == 0) {
                    // decode and sequence shards: the conv history before token 0
                    // comes from the tail
                    for (int e = tb; e < 3 * (kPP / 8); e += kGroupThreads) {
                        const int r = e / (kPP / 8), g = e % (kPP / 8);
                        *reinterpret_cast<uint4 *>(sm + kOffXbuf0 + r * (kPP * 2) + g * 16) =
                            *reinterpret_cast<const uint4 *>(p.tail + ((size_t)b * 4 + 1 + r) * ch +
                                                             hp * kPP + 8 * g);
                    }
                    grp_sync(2);
                }
                if (j < 2) head_rows(j);
                conv_chunk(j);
                grp_sync(2);
                if (tb == 0) {
                    tc::mbar_arrive(mb_xr);
                    tc::mbar_arrive(mb_free0 + 8 * (j & 1));   // (the conv reads no factors)
                }
            }
        } else {
            for (int j = 0; j < nk && ok; ++j) {
                ok = b_wait(mb_x0 + 8 * (j & 1), (j >> 1) & 1);
                if (!ok) break;
                if (j == 0 && !rev && p.tail && k0 == 0) {
                    // decode and sequence shards: the conv history before token 0
                    // comes from the tail
                    for (int e = tb; e < 3 * (kPP / 8); e += kGroupThreads) {
                        const int r = e / (kPP / 8), g = e % (kPP / 8);
                        *reinterpret_cast<uint4 *>(sm + kOffXbuf0 + r * (kPP * 2) + g * 16) =
                            *reinterpret_cast<const uint4 *>(p.tail + ((size_t)b * 4 + 1 + r) * ch +
                                                             hp * kPP + 8 * g);
                    }
                    grp_sync(2);
                }
                if (j < 2) head_rows(j);
                conv_chunk(j);
                if (j >= 1) {
                    // the state product of chunk j-1 has read wX
                    ok = b_wait(kStateOnly ? mb_e : mb_sdone, (j - 1) & 1);
                    if (!ok) break;
                }
                // (also the barrier between the conv's writes and wX's reads)
                ok = b_wait(mb_dt0 + 8 * (j & 1), (j >> 1) & 1);
                if (!ok) break;
                weight_chunk(j, tb);
                tc::fence_proxy_async();   // X and wX, for the tensor core
                grp_sync(2);
                if (tb == 0) {
                    tc::mbar_arrive(mb_s);
                    tc::mbar_arrive(mb_free0 + 8 * (j & 1));
                }
            }
        }
        if (!ok && tb == 0) record_error(p.status, kStatusTimeout);
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
    // L2 residency between the two directions' touches of a chunk (whole walks,
    // tied x, summed y): about 64 KB per kept chunk (its raw x and y rows),
    // kept for at most keep_dist walk steps, by every co-resident head pair,
    // within 100 MB of the 126 MB L2
    p.keep_dist = 0;
    if (sp.nseg == 1 && !pr.concat && xbc[0] == xbc[1]) {
        const long long pairs = std::min<long long>(kPlanSMs / 2, (long long)d.batch * (d.heads / kHeads));
        p.keep_dist = (int)std::min<long long>(p.nchunks, (100ll << 20) / (pairs * (64ll << 10)));
    }

    // prepass: B/C conv+SiLU in walk order for both directions
    bc_prepass_kernel<<<dim3((d.len + 31) / 32, d.batch, 2), 128, 0, stream>>>(
        xbc[0], xbc[1], p.tail, p.head, p.conv_w[0], p.conv_w[1], p.conv_b[0], p.conv_b[1], act, d.len,
        p.ch, d.heads * kP, d.batch);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();

    CUtensorMap tm_x_f, tm_x_r, tm_bc, tm_y;
    // y: (batch, len, H*P) summed, or (batch, len, 2*H*P) concatenated, stored by
    // 64-channel x 128-token boxes (the states-only launch stores nothing: its
    // map is a placeholder over the activations)
    const uint64_t ycols = (uint64_t)(pr.concat ? 2 : 1) * d.heads * kP;
    if (!make_map(&tm_x_f, xbc[0], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, kPP, kRawRows,
                  false) ||
        !make_map(&tm_x_r, xbc[1], (uint64_t)p.ch, (uint64_t)d.len, (uint64_t)d.batch, kPP, kRawRows,
                  false) ||
        !make_map(&tm_bc, act, (uint64_t)kBC, (uint64_t)d.len, (uint64_t)2 * d.batch, 64, kQ, true) ||
        !(p.y ? make_map(&tm_y, p.y, ycols, (uint64_t)d.len, (uint64_t)d.batch, kP, kQ, true)
              : make_map(&tm_y, act, (uint64_t)kBC, (uint64_t)d.len, (uint64_t)2 * d.batch, 64, kQ, true)))
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
        q.keep_dist = 0;
        ssd_tc_kernel<true, false><<<dim3(d.heads, d.batch, 1), kThreads, kSmemBytes, stream>>>(
            tm_x_f, tm_x_r, tm_bc, tm_y, q);
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
            tm_x_f, tm_x_r, tm_bc, tm_y, q);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        count_launch();
    }
    main_kernel<<<dim3(d.heads, d.batch, sp.nseg), kThreads, kSmemBytes, stream>>>(tm_x_f, tm_x_r, tm_bc,
                                                                                 tm_y, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    count_launch();
    if (ev.stop) e = cudaEventRecord(ev.stop, stream);
    return e;
}

}  // namespace bimamba
