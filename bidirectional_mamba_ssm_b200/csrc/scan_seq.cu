// scan_seq.cu -- token-sequential bidirectional selective scan on the CUDA
// cores (fp32 FMA), with the conv+SiLU fused into the staging step.
//
// This is the library's fp32 path: the tensor-core chunked path would have
// to round operands to bf16/tf32 and could not hold a 1e-4 relative bound,
// so fp32 activations are scanned here with fp32 state and fp32 math.
//
// Operation (Mamba-2 recurrence, per head h; "DiffuMamba" technical
// summaries, proposed-method sections; d_conv = 4 from the blog's
// network-architecture listing):
//     h_t = exp(dt_t A_h) h_{t-1} + dt_t x_t B_t^T ,   y_t = h_t C_t + D_h x_t
// run in walk order s = 0..len-1 for the forward stream (token s) and the
// reverse stream (token len-1-s, index reflection, no flip copy); the
// outputs are added.
//
// One CTA owns (batch b, head h, direction): the two directions run side by
// side and add their rows into y (zero-filled by the launcher; in fp32 a sum
// of two terms is exact in either order), or, with the concatenating fusion
// of untied directions, each writes its own half of each output row.  Each
// direction reads its own inputs and parameters.  Thread
// (p, q) owns state row p, columns n = q + NS*k (k < NPT), so each thread
// carries NPT fp32 state values in registers; the y dot product is reduced
// over the NS threads of a row with warp shuffles.  Activated x, B, C and dt
// of kChunk walk steps are staged in shared memory per chunk.
#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

constexpr int kSeqChunk = 32;

struct SeqParams {
    const void *xbc[2];     // [0] forward stream, [1] reverse stream
    const void *dt[2];
    const float *A[2];
    const float *D[2];
    const float *conv_w[2];
    const float *conv_b[2];
    int concat;        // y rows are [forward | reverse] (2*H*P wide)
    const void *tail;  // forward conv history (batch, 4, ch) or null
    const float *init;
    float *fin;
    void *y;
    int len, H, P, N, ch;
};

template <typename T, int NPT>
__global__ void __launch_bounds__(512)
scan_seq_kernel(SeqParams p)
{
    extern __shared__ float smem[];
    const int h = blockIdx.x, b = blockIdx.y, dir = blockIdx.z;
    const int P = p.P, N = p.N, H = p.H, len = p.len, ch = p.ch;
    const int NS = N / NPT;
    const int tid = threadIdx.x;
    const int row = tid / NS, q = tid % NS;
    float *xs = smem;                    // [kSeqChunk][P]
    float *bs = xs + kSeqChunk * P;      // [kSeqChunk][N]
    float *cs = bs + kSeqChunk * N;      // [kSeqChunk][N]
    float *ys = cs + kSeqChunk * N;      // [kSeqChunk][P]
    float *dts = ys + kSeqChunk * P;     // [kSeqChunk] dt
    float *as = dts + kSeqChunk;         // [kSeqChunk] exp(dt A)

    const T *tail = p.tail ? static_cast<const T *>(p.tail) + (size_t)b * 4 * ch : nullptr;
    const size_t ystride = (size_t)(p.concat ? 2 : 1) * H * P;   // y row length
    const int nch = P + 2 * N;
    // lanes present in this warp (the block need not be a multiple of 32)
    const int wbase = tid & ~31;
    const int nlanes = min(32, (int)blockDim.x - wbase);
    const unsigned lane_mask = nlanes == 32 ? 0xffffffffu : ((1u << nlanes) - 1u);
    const size_t sidx = ((size_t)b * H + h) * P * N;

    {
        const bool rev = dir == 1;
        // selects, not a run-time index into the parameter arrays
        const T *xbc = static_cast<const T *>(rev ? p.xbc[1] : p.xbc[0]) + (size_t)b * len * ch;
        const T *dtp = static_cast<const T *>(rev ? p.dt[1] : p.dt[0]) + (size_t)b * len * H;
        const float *conv_w = rev ? p.conv_w[1] : p.conv_w[0];
        const float *conv_b = rev ? p.conv_b[1] : p.conv_b[0];
        T *y = static_cast<T *>(p.y) + (size_t)b * len * ystride + (p.concat ? dir * H * P : 0);
        const float Ah = (rev ? p.A[1] : p.A[0])[h], Dh = (rev ? p.D[1] : p.D[0])[h];
        float st[NPT];
#pragma unroll
        for (int k = 0; k < NPT; ++k)
            st[k] = (!rev && p.init) ? p.init[sidx + (size_t)row * N + q + NS * k] : 0.0f;

        for (int s0 = 0; s0 < len; s0 += kSeqChunk) {
            const int cnt = min(kSeqChunk, len - s0);
            __syncthreads();
            // ---- stage conv+SiLU'd x (this head), B and C for cnt walk steps
            for (int ci = tid; ci < nch; ci += blockDim.x) {
                int c;
                float *dst;
                int dstride;
                if (ci < P) { c = h * P + ci; dst = xs + ci; dstride = P; }
                else if (ci < P + N) { c = H * P + (ci - P); dst = bs + (ci - P); dstride = N; }
                else { c = H * P + (ci - P); dst = cs + (ci - P - N); dstride = N; }
                auto raw = [&](int s) -> float {
                    if (s >= 0) return Elem<T>::load(xbc + (size_t)walk_token(s, len, rev) * ch + c);
                    if (!rev && tail) return Elem<T>::load(tail + (size_t)(4 + s) * ch + c);
                    return 0.0f;
                };
                if (conv_w) {
                    const float w0 = conv_w[c * 4 + 0], w1 = conv_w[c * 4 + 1];
                    const float w2 = conv_w[c * 4 + 2], w3 = conv_w[c * 4 + 3];
                    const float bias = conv_b ? conv_b[c] : 0.0f;
                    // 8 steps at a time, their raw values requested together
                    float r0 = raw(s0 - 3), r1 = raw(s0 - 2), r2 = raw(s0 - 1);
                    for (int i0 = 0; i0 < cnt; i0 += 8) {
                        float rv[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) rv[i] = i0 + i < cnt ? raw(s0 + i0 + i) : 0.0f;
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            if (i0 + i >= cnt) break;
                            float acc = bias;
                            acc = fmaf(w0, r0, acc);
                            acc = fmaf(w1, r1, acc);
                            acc = fmaf(w2, r2, acc);
                            acc = fmaf(w3, rv[i], acc);
                            dst[(i0 + i) * dstride] = silu_f(acc);
                            r0 = r1; r1 = r2; r2 = rv[i];
                        }
                    }
                } else {
                    for (int i = 0; i < cnt; ++i) dst[i * dstride] = raw(s0 + i);
                }
            }
            for (int i = tid; i < cnt; i += blockDim.x) {
                const float dv = Elem<T>::load(dtp + (size_t)walk_token(s0 + i, len, rev) * H + h);
                dts[i] = dv;
                as[i] = expf(dv * Ah);
            }
            __syncthreads();

            // ---- recurrence over the chunk
#pragma unroll 4
            for (int i = 0; i < cnt; ++i) {
                const float d = dts[i];
                const float a = as[i];
                const float xv = xs[i * P + row];
                const float dx = d * xv;
                const float *bi = bs + i * N + q;
                const float *cI = cs + i * N + q;
                float acc = 0.0f;
#pragma unroll
                for (int k = 0; k < NPT; ++k) {
                    st[k] = fmaf(a, st[k], dx * bi[NS * k]);
                    acc = fmaf(st[k], cI[NS * k], acc);
                }
                for (int off = NS >> 1; off > 0; off >>= 1)
                    acc += __shfl_xor_sync(lane_mask, acc, off);
                if (q == 0) ys[i * P + row] = fmaf(Dh, xv, acc);
            }
            __syncthreads();

            // ---- write back: added into the zero-filled y (sum fusion), or
            // stored into this direction's half of the row (concatenation)
            for (int e = tid; e < cnt * P; e += blockDim.x) {
                const int i = e / P, pc = e % P;
                T *yp = y + (size_t)walk_token(s0 + i, len, rev) * ystride + h * P + pc;
                if (p.concat)
                    Elem<T>::store(yp, ys[e]);
                else
                    atomicAdd(yp, static_cast<T>(ys[e]));
            }
        }
        if (!rev && p.fin) {
#pragma unroll
            for (int k = 0; k < NPT; ++k) p.fin[sidx + (size_t)row * N + q + NS * k] = st[k];
        }
    }
}

template <typename T, int NPT>
static cudaError_t launch_seq_t(const SeqParams &p, int batch, cudaStream_t stream)
{
    const int threads = p.P * (p.N / NPT);
    const size_t smem = sizeof(float) * (size_t)(kSeqChunk * (2 * p.P + 2 * p.N) + 2 * kSeqChunk);
    cudaError_t e = cudaFuncSetAttribute(scan_seq_kernel<T, NPT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const TimingEvents ev = timing_events();
    if (ev.start && (e = cudaEventRecord(ev.start, stream)) != cudaSuccess) return e;
    // the directions add their rows into y
    if (!p.concat &&
        (e = cudaMemsetAsync(p.y, 0, (size_t)batch * p.len * p.H * p.P * sizeof(T), stream)) != cudaSuccess)
        return e;
    scan_seq_kernel<T, NPT><<<dim3(p.H, batch, 2), threads, smem, stream>>>(p);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    count_launch();
    if (ev.stop) err = cudaEventRecord(ev.stop, stream);
    return err;
}

template <typename T>
cudaError_t launch_scan_seq(const Problem &pr, cudaStream_t stream)
{
    const bimamba_dims &d = pr.dims;
    const int batch = d.batch, len = d.len, H = d.heads, P = d.headdim, N = d.d_state;
    SeqParams p{};
    for (int i = 0; i < 2; ++i) {
        p.xbc[i] = pr.xbc[i]; p.dt[i] = pr.dt[i]; p.A[i] = pr.A[i]; p.D[i] = pr.D[i];
        p.conv_w[i] = pr.conv_w[i]; p.conv_b[i] = pr.conv_b[i];
    }
    p.concat = pr.concat;
    p.tail = pr.tail;
    p.init = pr.init;
    p.fin = pr.fin;
    p.y = pr.y;
    p.len = len; p.H = H; p.P = P; p.N = N; p.ch = H * P + 2 * N;
    // at most 512 threads per CTA: P * (N / NPT) <= 512 for P <= 128, N <= 256
    if (N >= 64 && P * (N / 32) > 512) return launch_seq_t<T, 64>(p, batch, stream);
    if (N >= 32) return launch_seq_t<T, 32>(p, batch, stream);
    if (N == 16) return launch_seq_t<T, 4>(p, batch, stream);
    return launch_seq_t<T, 8>(p, batch, stream);
}

template cudaError_t launch_scan_seq<float>(const Problem &, cudaStream_t);
template cudaError_t launch_scan_seq<__nv_bfloat16>(const Problem &, cudaStream_t);

// tail_out[s][k] = (prefix | block)[len - 4 + k], oldest first.
template <typename T>
__global__ void tail_commit_kernel(const T *__restrict__ block, const T *__restrict__ tail,
                                   T *__restrict__ tail_out, int len, int ch)
{
    const int s = blockIdx.y, k = blockIdx.z;
    const int pos = len - 4 + k;
    const T *src = pos >= 0 ? block + ((size_t)s * len + pos) * ch
                            : tail + ((size_t)s * 4 + (4 + pos)) * ch;
    T *dst = tail_out + ((size_t)s * 4 + k) * ch;
    for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < ch; c += gridDim.x * blockDim.x)
        dst[c] = src[c];
}

template <typename T>
cudaError_t launch_tail_commit(const void *block, const void *tail, void *tail_out, int streams,
                               int len, int ch, cudaStream_t stream)
{
    dim3 grid((ch + 255) / 256, streams, 4);
    tail_commit_kernel<T><<<grid, 256, 0, stream>>>(static_cast<const T *>(block),
                                                    static_cast<const T *>(tail),
                                                    static_cast<T *>(tail_out), len, ch);
    cudaError_t err = cudaGetLastError();
    if (err == cudaSuccess) count_launch();
    return err;
}

template cudaError_t launch_tail_commit<float>(const void *, const void *, void *, int, int, int,
                                               cudaStream_t);
template cudaError_t launch_tail_commit<__nv_bfloat16>(const void *, const void *, void *, int,
                                                       int, int, cudaStream_t);

}  // namespace bimamba
