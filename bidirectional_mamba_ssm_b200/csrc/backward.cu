// backward.cu -- gradients of the bidirectional mixer core (training path).
//
// The mixer core is y = scan_fwd(conv_fwd(xbc)) + scan_rev(conv_rev(xbc))
// ("DiffuMamba: High-Throughput Diffusion LMs with Mamba Backbone",
// technical summaries section 2: a bidirectional Mamba-2 mixer, forward and
// reverse streams added, trained with the masked-diffusion objective; the
// Mamba-2 recurrence h_t = exp(dt_t A) h_{t-1} + dt_t x_t B_t^T,
// y_t = h_t C_t + D x_t).  Given dy = dL/dy this computes dL/d(xbc, dt, A,
// D, conv taps, conv bias, initial state), in fp32.
//
// Pipeline (per call):
//  1. the activated xBC of both streams (conv + SiLU; the stand-alone conv
//     kernel, in the activation dtype);
//  2. bwd_state_kernel, one CTA per (sequence, head, direction): the state
//     entering every chunk of Q = 64 walk steps, S_{k+1} = e^{c_last} S_k +
//     X^T diag(w) B, kept in the workspace;
//  3. bwd_scan_kernel, one CTA per (sequence, head, direction), chunks from
//     the last: with W[t,s] = (C_t.B_s) e^{c_t-c_s} dt_s and T[t,s] =
//     (dY_t.x_s) e^{c_t-c_s} dt_s (s <= t), w_s = e^{c_last-c_s} dt_s, the
//     state S_in entering the chunk and dS the adjoint of the state leaving it
//         dX = W^T dY + D dY + w o (B dS^T)
//         dB = T^T C + w o (X dS)          (summed over heads: one group)
//         dC = T B + e^c o (dY S_in)
//         dS_in = e^{c_last} dS + (e^c o dY)^T C
//     and dt, A through dL/dc_j of the chunk's prefix sums (suffix sums for
//     dt, sum_j dL/dc_j sum_{i<=j} dt_i for A); the small matrix products run
//     on the CUDA cores out of shared memory;
//  4. bwd_conv_staged_kernel (conv_staged.cu): each stream's dact through
//     SiLU' and the transposed taps to d(xbc), plus the tap and bias
//     gradients, both streams at once.
#include <algorithm>

#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

namespace {

constexpr int kBQ = 64;          // chunk length of the backward
constexpr int kBThreads = 256;

// C (M x N) = sum_k a(m, k) b(k, n) over the CTA's 256 threads.  A thread
// owns rows m0 .. m0+TM-1 and the TN columns n0 + j cs (cs = N / TN), so
// that the threads of a warp read consecutive columns of b (no bank
// conflicts on a row-major b); `put(m0, n0, cs, acc)` stores the tile,
// acc[i][j] being element (m0 + i, n0 + j cs).
template <int TM, int TN, typename FA, typename FB, typename FP>
__device__ __forceinline__ void mm(int M, int N, int K, FA a, FB b, FP put)
{
    const int cs = N / TN;
    const int ntiles = (M / TM) * cs;
    for (int tile = threadIdx.x; tile < ntiles; tile += kBThreads) {
        const int m0 = (tile / cs) * TM, n0 = tile % cs;
        float acc[TM][TN];
#pragma unroll
        for (int i = 0; i < TM; ++i)
#pragma unroll
            for (int j = 0; j < TN; ++j) acc[i][j] = 0.0f;
        for (int k = 0; k < K; ++k) {
            float av[TM], bv[TN];
#pragma unroll
            for (int i = 0; i < TM; ++i) av[i] = a(m0 + i, k);
#pragma unroll
            for (int j = 0; j < TN; ++j) bv[j] = b(k, n0 + j * cs);
#pragma unroll
            for (int i = 0; i < TM; ++i)
#pragma unroll
                for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        put(m0, n0, cs, acc);
    }
}

__device__ __forceinline__ float block_sum(float v, float *red)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float s = 0.0f;
#pragma unroll
    for (int i = 0; i < kBThreads / 32; ++i) s += red[i];
    return s;
}

struct BwdParams {
    const void *act[2];     // (batch, len, ch) activated xBC of the forward / reverse stream
    const void *dt;         // (batch, len, H)
    const void *dy;         // (batch, len, H*P)
    const float *A, *D, *init;
    float *states;          // [dir][batch][H][nchunks][P][N]: state entering each chunk
    float *dact[2];         // (batch, len, ch) fp32 per stream (x part written, B/C accumulated)
    float *ddt, *dA, *dD, *dinit;
    int batch, len, H, P, N, ch, nchunks;
};

template <typename T>
__device__ __forceinline__ float ldv(const void *p, size_t i)
{
    return Elem<T>::load(static_cast<const T *>(p) + i);
}

}  // namespace

// dynamic shared memory of the chunked backward, in floats
static size_t bwd_smem_floats(int P, int N)
{
    return (size_t)2 * kBQ * P      // X, dY
           + 2 * kBQ * N            // B, C
           + (size_t)P * N          // dS
           + 2 * kBQ * kBQ          // W, T
           + 2 * kBQ * N            // X dS, dY S_in
           + 9 * kBQ + 64;          // per-slot vectors, reductions
}

static size_t bwd_state_smem_floats(int P, int N)
{
    return (size_t)kBQ * P + (size_t)kBQ * N + (size_t)P * N + kBQ;
}

// The state entering every chunk of one (sequence, head, direction) walk.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_state_kernel(const BwdParams p)
{
    extern __shared__ float fs[];
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    const bool rev = dir != 0;
    const int P = p.P, N = p.N, L = p.len, H = p.H, ch = p.ch;
    float *X = fs;                      // [Q][P]  w-scaled
    float *Bs = X + kBQ * P;            // [Q][N]
    float *S = Bs + kBQ * N;            // [P][N]
    float *cvec = S + P * N;            // [Q]
    const void *act = rev ? p.act[1] : p.act[0];
    const size_t pn = (size_t)P * N;
    float *out = p.states + ((((size_t)dir * p.batch + b) * H + h) * p.nchunks) * pn;
    const float Ah = p.A[h];
    for (int i = threadIdx.x; i < P * N; i += kBThreads)
        S[i] = (!rev && p.init) ? p.init[((size_t)b * H + h) * pn + i] : 0.0f;
    __syncthreads();
    for (int k = 0; k < p.nchunks; ++k) {
        for (int i = threadIdx.x; i < P * N; i += kBThreads) out[(size_t)k * pn + i] = S[i];
        const int s0 = k * kBQ, cnt = min(kBQ, L - s0);
        if (threadIdx.x < 32) {
            // prefix sums of dt*A over the chunk (natural units)
            float run = 0.0f;
            for (int j = 0; j < kBQ; j += 32) {
                const int jj = j + threadIdx.x;
                const int tok = rev ? L - 1 - (s0 + jj) : s0 + jj;
                float v = jj < cnt ? ldv<T>(p.dt, (size_t)(b * L + tok) * H + h) * Ah : 0.0f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, v, o);
                    if ((int)threadIdx.x >= o) v += u;
                }
                cvec[jj] = run + v;
                run += __shfl_sync(0xffffffffu, v, 31);
            }
        }
        __syncthreads();
        const float clast = cvec[cnt - 1];
        for (int i = threadIdx.x; i < kBQ * P; i += kBThreads) {
            const int j = i / P, q = i % P;
            float v = 0.0f;
            if (j < cnt) {
                const int tok = rev ? L - 1 - (s0 + j) : s0 + j;
                const float d = ldv<T>(p.dt, (size_t)(b * L + tok) * H + h);
                v = ldv<T>(act, ((size_t)b * L + tok) * ch + h * P + q) * expf(clast - cvec[j]) * d;
            }
            X[i] = v;
        }
        for (int i = threadIdx.x; i < kBQ * N; i += kBThreads) {
            const int j = i / N, n = i % N;
            float v = 0.0f;
            if (j < cnt) {
                const int tok = rev ? L - 1 - (s0 + j) : s0 + j;
                v = ldv<T>(act, ((size_t)b * L + tok) * ch + H * P + n);
            }
            Bs[i] = v;
        }
        __syncthreads();
        const float al = expf(clast);
        // S = e^{c_last} S + X^T B  (P x N, K = Q)
        mm<4, 4>(P, N, kBQ, [&](int m, int kk) { return X[kk * P + m]; },
                 [&](int kk, int n) { return Bs[kk * N + n]; },
                 [&](int m0, int n0, int cs, float (&acc)[4][4]) {
                     for (int i = 0; i < 4; ++i)
                         for (int j = 0; j < 4; ++j) {
                             float &s = S[(m0 + i) * N + n0 + j * cs];
                             s = fmaf(al, s, acc[i][j]);
                         }
                 });
        __syncthreads();
    }
}

// The chunked backward of one (sequence, head, direction) walk.
template <typename T>
__global__ void __launch_bounds__(kBThreads)
bwd_scan_kernel(const BwdParams p)
{
    extern __shared__ float fs[];
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    const bool rev = dir != 0;
    const int P = p.P, N = p.N, L = p.len, H = p.H, ch = p.ch;
    float *X = fs;                    // [Q][P]
    float *dY = X + kBQ * P;          // [Q][P]
    float *Bs = dY + kBQ * P;         // [Q][N]
    float *Cs = Bs + kBQ * N;         // [Q][N]
    float *dS = Cs + kBQ * N;         // [P][N]  adjoint of the state leaving the chunk
    float *Wm = dS + P * N;           // [Q][Q]
    float *Tm = Wm + kBQ * kBQ;       // [Q][Q]
    float *XdS = Tm + kBQ * kBQ;      // [Q][N]  X dS
    float *dYS = XdS + kBQ * N;       // [Q][N]  dY S_in
    float *cvec = dYS + kBQ * N;      // [Q] prefix sums c
    float *dtv = cvec + kBQ;          // [Q] dt
    float *rsum = dtv + kBQ;          // [Q] row sums of DYX o W
    float *csum = rsum + kBQ;         // [Q] column sums of DYX o W
    float *ddt = csum + kBQ;          // [Q] direct dt terms
    float *dc = ddt + kBQ;            // [Q] dL/dc
    float *U = dc + kBQ;              // [Q]
    float *ecv = U + kBQ;             // [Q] e^{c_t} (0 past the chunk end)
    float *red = ecv + kBQ;           // reductions (+ 2 * kBQ spare)
    // X, B and dS are also read down their columns (by consecutive threads):
    // element (r, c) of each is stored at column c ^ (r & m) of row r, m + 1
    // = the largest power of two (at most 32) dividing the row length, so
    // that the column stays in its row and both rows and columns spread over
    // the banks
    const int mP = min(P & -P, 32) - 1, mN = min(N & -N, 32) - 1;
    auto swx = [mP](int r, int c) { return c ^ (r & mP); };   // X [Q][P]
    auto sw = [mN](int r, int c) { return c ^ (r & mN); };    // B [Q][N], dS [P][N]
    const void *act = rev ? p.act[1] : p.act[0];
    float *dact = rev ? p.dact[1] : p.dact[0];
    const size_t pn = (size_t)P * N;
    const float *states = p.states + ((((size_t)dir * p.batch + b) * H + h) * p.nchunks) * pn;
    const float Ah = p.A[h], Dh = p.D[h];
    const int tid = threadIdx.x, lane = tid & 31;
    float dA_acc = 0.0f, dD_acc = 0.0f;
    for (int i = tid; i < P * N; i += kBThreads) dS[i] = 0.0f;   // (zero in any layout)
    for (int k = p.nchunks - 1; k >= 0; --k) {
        const int s0 = k * kBQ, cnt = min(kBQ, L - s0);
        const float *Sin = states + (size_t)k * pn;   // read from L2
        auto tok_of = [&](int j) { return rev ? L - 1 - (s0 + j) : s0 + j; };
        // ---- the chunk's operands
        for (int i = tid; i < kBQ * P; i += kBThreads) {
            const int j = i / P, q = i % P;
            float xv = 0.0f, gv = 0.0f;
            if (j < cnt) {
                const size_t ti = (size_t)b * L + tok_of(j);
                xv = ldv<T>(act, ti * ch + h * P + q);
                gv = ldv<T>(p.dy, ti * (size_t)H * P + h * P + q);
            }
            X[j * P + swx(j, q)] = xv;
            dY[i] = gv;
        }
        for (int i = tid; i < kBQ * N; i += kBThreads) {
            const int j = i / N, n = i % N;
            float bv = 0.0f, cv = 0.0f;
            if (j < cnt) {
                const size_t ti = (size_t)b * L + tok_of(j);
                bv = ldv<T>(act, ti * ch + H * P + n);
                cv = ldv<T>(act, ti * ch + H * P + N + n);
            }
            Bs[j * N + sw(j, n)] = bv;
            Cs[i] = cv;
        }
        if (tid < kBQ) {
            rsum[tid] = 0.0f;
            csum[tid] = 0.0f;
            ddt[tid] = 0.0f;
        }
        if (tid < 32) {
            float run = 0.0f;
            for (int j = 0; j < kBQ; j += 32) {
                const int jj = j + tid;
                const float d = jj < cnt ? ldv<T>(p.dt, (size_t)(b * L + tok_of(jj)) * H + h) : 0.0f;
                float v = d * Ah;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const float u = __shfl_up_sync(0xffffffffu, v, o);
                    if (tid >= o) v += u;
                }
                cvec[jj] = run + v;
                dtv[jj] = d;
                run += __shfl_sync(0xffffffffu, v, 31);
            }
        }
        __syncthreads();
        const float clast = cvec[cnt - 1];
        // ---- CB = C B^T, DYX = dY X^T (Q x Q), then W, T and the sums of their products
        mm<4, 4>(kBQ, kBQ, N, [&](int t, int n) { return Cs[t * N + n]; },
                 [&](int n, int s) { return Bs[s * N + sw(s, n)]; },
                 [&](int t0, int u0, int cs, float (&acc)[4][4]) {
                     for (int i = 0; i < 4; ++i)
                         for (int j = 0; j < 4; ++j) Wm[(t0 + i) * kBQ + u0 + j * cs] = acc[i][j];
                 });
        mm<4, 4>(kBQ, kBQ, P, [&](int t, int q) { return dY[t * P + q]; },
                 [&](int q, int s) { return X[s * P + swx(s, q)]; },
                 [&](int t0, int u0, int cs, float (&acc)[4][4]) {
                     for (int i = 0; i < 4; ++i)
                         for (int j = 0; j < 4; ++j) Tm[(t0 + i) * kBQ + u0 + j * cs] = acc[i][j];
                 });
        // ---- X dS and dY S_in (Q x N, K = P)
        mm<2, 4>(kBQ, N, P, [&](int s, int q) { return X[s * P + swx(s, q)]; },
                 [&](int q, int n) { return dS[q * N + sw(q, n)]; },
                 [&](int m0, int n0, int cs, float (&acc)[2][4]) {
                     for (int i = 0; i < 2; ++i)
                         for (int j = 0; j < 4; ++j) XdS[(m0 + i) * N + n0 + j * cs] = acc[i][j];
                 });
        mm<2, 4>(kBQ, N, P, [&](int t, int q) { return dY[t * P + q]; },
                 [&](int q, int n) { return Sin[q * N + n]; },
                 [&](int m0, int n0, int cs, float (&acc)[2][4]) {
                     for (int i = 0; i < 2; ++i)
                         for (int j = 0; j < 4; ++j) dYS[(m0 + i) * N + n0 + j * cs] = acc[i][j];
                 });
        __syncthreads();
        // element (t, s), s <= t: e = e^{c_t - c_s}, W = CB e dt_s, T = DYX e dt_s;
        // dL/dc gets the row sums minus the column sums of DYX o W, dt_s the
        // column sums of DYX o CB o e.  A warp covers 32 s of one row t.
        for (int i = tid; i < kBQ * kBQ; i += kBThreads) {
            const int t = i / kBQ, s = i % kBQ;
            float w = 0.0f, tt = 0.0f, tw = 0.0f;
            if (s <= t && t < cnt) {
                const float e = expf(fminf(cvec[t] - cvec[s], 0.0f));
                const float cb = Wm[i], dyx = Tm[i], d = dtv[s];
                w = cb * e * d;
                tt = dyx * e * d;
                tw = dyx * w;
                atomicAdd(ddt + s, dyx * cb * e);
                atomicAdd(csum + s, tw);
            }
            Wm[i] = w;
            Tm[i] = tt;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) tw += __shfl_xor_sync(0xffffffffu, tw, o);
            if (lane == 0) atomicAdd(rsum + t, tw);
        }
        // per slot: U_s = w_s (x_s^T dS B_s), the off-diagonal term of dc, the
        // state's direct dt term
        for (int j = tid; j < kBQ; j += kBThreads) {
            float xb = 0.0f, cs = 0.0f;
            for (int n = 0; n < N; ++n) {
                xb = fmaf(XdS[j * N + n], Bs[j * N + sw(j, n)], xb);
                cs = fmaf(Cs[j * N + n], dYS[j * N + n], cs);
            }
            const bool in = j < cnt;
            const float el = in ? expf(clast - cvec[j]) : 0.0f;
            ecv[j] = in ? expf(cvec[j]) : 0.0f;
            U[j] = el * dtv[j] * xb;
            dc[j] = in ? expf(cvec[j]) * cs - U[j] : 0.0f;
            red[kBQ + j] = el * xb;   // direct dt term of the state
        }
        __syncthreads();
        // ---- dX = W^T dY + D dY + w o (B dS^T)   (Q x P)
        mm<2, 4>(kBQ, P, kBQ, [&](int s, int t) { return Wm[t * kBQ + s]; },
                 [&](int t, int q) { return dY[t * P + q]; },
                 [&](int m0, int q0, int cs, float (&acc)[2][4]) {
                     for (int i = 0; i < 2; ++i) {
                         const int s = m0 + i;
                         if (s >= cnt) continue;
                         float bds[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                         for (int n = 0; n < N; ++n) {
                             const float bv = Bs[s * N + sw(s, n)];
#pragma unroll
                             for (int j = 0; j < 4; ++j) {
                                 const int q = q0 + j * cs;
                                 bds[j] = fmaf(bv, dS[q * N + sw(q, n)], bds[j]);
                             }
                         }
                         const float wl = expf(clast - cvec[s]) * dtv[s];
                         const size_t ti = (size_t)b * L + tok_of(s);
                         for (int j = 0; j < 4; ++j) {
                             const int q = q0 + j * cs;
                             dact[ti * ch + h * P + q] = acc[i][j] + Dh * dY[s * P + q] + wl * bds[j];
                         }
                     }
                 });
        // ---- dB = T^T C + w o (X dS);  dC = T B + e^c o (dY S_in)   (Q x N, summed over heads)
        mm<2, 4>(kBQ, N, kBQ, [&](int s, int t) { return Tm[t * kBQ + s]; },
                 [&](int t, int n) { return Cs[t * N + n]; },
                 [&](int m0, int n0, int cs, float (&acc)[2][4]) {
                     for (int i = 0; i < 2; ++i) {
                         const int s = m0 + i;
                         if (s >= cnt) continue;
                         const float wl = expf(clast - cvec[s]) * dtv[s];
                         const size_t ti = (size_t)b * L + tok_of(s);
                         for (int j = 0; j < 4; ++j) {
                             const int n = n0 + j * cs;
                             atomicAdd(dact + ti * ch + H * P + n, acc[i][j] + wl * XdS[s * N + n]);
                         }
                     }
                 });
        mm<2, 4>(kBQ, N, kBQ, [&](int t, int s) { return Tm[t * kBQ + s]; },
                 [&](int s, int n) { return Bs[s * N + sw(s, n)]; },
                 [&](int m0, int n0, int cs, float (&acc)[2][4]) {
                     for (int i = 0; i < 2; ++i) {
                         const int t = m0 + i;
                         if (t >= cnt) continue;
                         const float ec = ecv[t];
                         const size_t ti = (size_t)b * L + tok_of(t);
                         for (int j = 0; j < 4; ++j) {
                             const int n = n0 + j * cs;
                             atomicAdd(dact + ti * ch + H * P + N + n, acc[i][j] + ec * dYS[t * N + n]);
                         }
                     }
                 });
        // ---- dL/dc, then dt (suffix sums), A and D
        float sdS = 0.0f;   // <dS, S_in>
        for (int i = tid; i < P * N; i += kBThreads) sdS = fmaf(dS[(i / N) * N + sw(i / N, i % N)], Sin[i], sdS);
        sdS = block_sum(sdS, red);
        float dd = 0.0f;
        for (int i = tid; i < cnt * P; i += kBThreads) dd = fmaf(dY[i], X[(i / P) * P + swx(i / P, i % P)], dd);
        dD_acc += block_sum(dd, red);
        if (tid == 0) {
            float usum = 0.0f;
            for (int j = 0; j < cnt; ++j) usum += U[j];
            for (int j = 0; j < cnt; ++j) dc[j] += rsum[j] - csum[j];
            dc[cnt - 1] += expf(clast) * sdS + usum;
            float suffix = 0.0f, cum = 0.0f;
            for (int j = cnt - 1; j >= 0; --j) {
                suffix += dc[j];
                const float g = ddt[j] + red[kBQ + j] + Ah * suffix;
                atomicAdd(p.ddt + (size_t)(b * L + tok_of(j)) * H + h, g);
            }
            for (int j = 0; j < cnt; ++j) {
                cum += dtv[j];
                dA_acc = fmaf(dc[j], cum, dA_acc);
            }
        }
        __syncthreads();   // every product that reads dS is done
        // ---- dS_in = e^{c_last} dS + (e^c o dY)^T C   (P x N, K = Q), in place
        const float al = expf(clast);
        mm<4, 4>(P, N, kBQ, [&](int q, int t) { return ecv[t] * dY[t * P + q]; },
                 [&](int t, int n) { return Cs[t * N + n]; },
                 [&](int q0, int n0, int cs, float (&acc)[4][4]) {
                     for (int i = 0; i < 4; ++i)
                         for (int j = 0; j < 4; ++j) {
                             const int q = q0 + i, n = n0 + j * cs;
                             float &v = dS[q * N + sw(q, n)];
                             v = fmaf(al, v, acc[i][j]);
                         }
                 });
        __syncthreads();
    }
    if (tid == 0) {
        atomicAdd(p.dA + h, dA_acc);
        atomicAdd(p.dD + h, dD_acc);
    }
    if (!rev && p.dinit)
        for (int i = tid; i < P * N; i += kBThreads)
            p.dinit[((size_t)b * H + h) * pn + i] = dS[(i / N) * N + sw(i / N, i % N)];
}

bool backward_supported(const bimamba_dims &d)
{
    return d.ngroups == 1 && d.d_conv == 4 && d.headdim <= 64 && d.d_state <= 128 &&
           d.headdim % 4 == 0 && d.d_state % 4 == 0;
}

size_t backward_workspace_bytes(const bimamba_dims &d)
{
    const size_t esz = d.dtype == BIMAMBA_F32 ? 4 : 2;
    const size_t ch = (size_t)d.heads * d.headdim + 2 * d.d_state;
    const size_t tokens = (size_t)d.batch * d.len;
    const size_t nchunks = ((size_t)d.len + kBQ - 1) / kBQ;
    const size_t act = (2 * tokens * ch * esz + 255) & ~(size_t)255;
    const size_t dact = 2 * tokens * ch * sizeof(float);
    const size_t states = 2 * (size_t)d.batch * d.heads * nchunks * d.headdim * d.d_state * sizeof(float);
    return act + dact + std::max(states, backward_tc_supported(d) ? backward_tc_state_bytes(d) : (size_t)0);
}

template <typename T>
cudaError_t launch_backward_t(const BackwardProblem &q, cudaStream_t s)
{
    const bimamba_dims &d = q.dims;
    const int ch = d.heads * d.headdim + 2 * d.d_state;
    const size_t tokens = (size_t)d.batch * d.len;
    const size_t esz = sizeof(T);
    char *ws = static_cast<char *>(q.workspace);
    BwdParams p;
    p.act[0] = ws;
    p.act[1] = ws + tokens * ch * esz;
    const size_t act = (2 * tokens * ch * esz + 255) & ~(size_t)255;
    p.dact[0] = reinterpret_cast<float *>(ws + act);
    p.dact[1] = p.dact[0] + tokens * ch;
    p.states = p.dact[1] + tokens * ch;
    p.dt = q.dt;
    p.dy = q.dy;
    p.A = q.A;
    p.D = q.D;
    p.init = q.init;
    p.ddt = q.ddt;
    p.dA = q.dA;
    p.dD = q.dD;
    p.dinit = q.dinit;
    p.batch = d.batch;
    p.len = d.len;
    p.H = d.heads;
    p.P = d.headdim;
    p.N = d.d_state;
    p.ch = ch;
    p.nchunks = (d.len + kBQ - 1) / kBQ;
    cudaError_t e;
    // outputs that are accumulated start at zero.  Of the two streams' fp32
    // activation gradients (contiguous rows of ch), the tensor-core passes
    // overwrite the x columns of every row and add to the B/C columns: only
    // those are zeroed there (a strided 2-D fill), the whole rows otherwise
    const bool tc_path = backward_tc_supported(d);
    e = tc_path ? cudaMemset2DAsync(p.dact[0] + (size_t)d.heads * d.headdim, ch * sizeof(float), 0,
                                    (size_t)2 * d.d_state * sizeof(float), 2 * tokens, s)
                : cudaMemsetAsync(p.dact[0], 0, 2 * tokens * ch * sizeof(float), s);
    if (e != cudaSuccess ||
        (e = cudaMemsetAsync(q.ddt, 0, tokens * d.heads * sizeof(float), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(q.dA, 0, d.heads * sizeof(float), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(q.dD, 0, d.heads * sizeof(float), s)) != cudaSuccess ||
        (e = cudaMemsetAsync(q.dconv_w, 0, (size_t)ch * 4 * sizeof(float), s)) != cudaSuccess ||
        (q.dconv_b && (e = cudaMemsetAsync(q.dconv_b, 0, (size_t)ch * sizeof(float), s)) != cudaSuccess))
        return e;
    // both streams' activations from one pass over the raw rows (TMA-staged
    // tiles; the entry point has checked the 16-byte alignment they need)
    if ((e = launch_conv_silu_both_staged<T>(q.xbc, const_cast<void *>(p.act[0]), const_cast<void *>(p.act[1]),
                                             q.conv_w, q.conv_b, d.batch, d.len, ch, s)) != cudaSuccess)
        return e;
    if (tc_path) {
        // the state and adjoint passes on the tensor cores
        BackwardTcProblem t{};
        t.dims = d;
        t.act[0] = p.act[0];
        t.act[1] = p.act[1];
        t.dt = q.dt;
        t.dy = q.dy;
        t.A = q.A;
        t.D = q.D;
        t.init = q.init;
        t.dact[0] = p.dact[0];
        t.dact[1] = p.dact[1];
        t.ddt = q.ddt;
        t.dA = q.dA;
        t.dD = q.dD;
        t.dinit = q.dinit;
        t.states = p.states;
        if ((e = launch_backward_tc(t, s)) != cudaSuccess) return e;
    } else {
        const size_t smem = bwd_smem_floats(d.headdim, d.d_state) * sizeof(float);
        const size_t smem_st = bwd_state_smem_floats(d.headdim, d.d_state) * sizeof(float);
        if ((e = cudaFuncSetAttribute(bwd_state_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem_st)) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_scan_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        const dim3 grid(d.heads, d.batch, 2);
        bwd_state_kernel<T><<<grid, kBThreads, smem_st, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch();
        const TimingEvents ev = timing_events();
        if (ev.start && (e = cudaEventRecord(ev.start, s)) != cudaSuccess) return e;
        bwd_scan_kernel<T><<<grid, kBThreads, smem, s>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch();
        if (ev.stop && (e = cudaEventRecord(ev.stop, s)) != cudaSuccess) return e;
    }
    return launch_bwd_conv_staged<T>(q.xbc, q.conv_w, q.conv_b, p.dact[0], p.dact[1], q.dxbc, q.dconv_w,
                                     q.dconv_b, d.batch, d.len, ch, s);
}

cudaError_t launch_backward(const BackwardProblem &q, cudaStream_t s)
{
    return q.dims.dtype == BIMAMBA_F32 ? launch_backward_t<float>(q, s)
                                       : launch_backward_t<__nv_bfloat16>(q, s);
}

}  // namespace bimamba
