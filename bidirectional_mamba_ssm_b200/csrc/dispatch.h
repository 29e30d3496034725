// dispatch.h -- internal launcher declarations of the mixer library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/bimamba.h"

namespace bimamba {

// One validated call of the bidirectional mixer core (full scan or decode).
// Per-direction inputs: [0] the forward stream, [1] the reverse stream (the
// same pointers when the directions share their parameters).
struct Problem {
    bimamba_dims dims;
    const void *xbc[2];
    const void *dt[2];
    const float *A[2];
    const float *D[2];
    const float *conv_w[2];   // null: xbc already activated
    const float *conv_b[2];
    int concat;            // 0: y = forward + reverse; 1: y = [forward | reverse] per token
    const void *tail;      // forward conv history (decode, sequence shards) or null
    const void *head;      // raw tokens after a sequence shard (reverse conv) or null
    // sequence shards: all ranks' shard end states and log2 decays, this rank
    const float *shard_states;
    const float *shard_dec;
    int rank, nranks;
    // states-only call: write this shard's end states / decays, no outputs
    float *states_out;
    float *dec_out;
    const float *init;     // forward initial state or null
    float *fin;            // forward final state or null
    void *y;
    void *workspace;
    size_t workspace_bytes;
    int *status;           // device status word
};

size_t workspace_bytes_for(const bimamba_dims &d);
// argument checks of bimamba_block_decode (nothing launched); BIMAMBA_OK or an error
int check_block_decode(const bimamba_dims *d, const void *xbc_block, const void *dt_block,
                       const float *A, const float *D, const float *conv_w, const float *conv_b,
                       const float *state, const void *tail, const void *y, const float *state_out,
                       const void *tail_out);
cudaError_t launch_bimamba(const Problem &p, cudaStream_t stream);

// chunked tensor-core path (bf16, headdim 64, d_state 128)
bool tc_path_supported(const bimamba_dims &d);
size_t tc_workspace_bytes(const bimamba_dims &d);
// leading bytes of that workspace that must be zero when a call starts (the
// forward/reverse meeting counters); the rest is rewritten by every call
size_t tc_counter_bytes(const bimamba_dims &d);
// out[0..2]: segments per direction, chunks per segment, state-only items
void tc_launch_plan(const bimamba_dims &d, int *out);
cudaError_t launch_ssd_tc(const Problem &p, cudaStream_t stream);
// end states from zero and log2 decays of a whole sequence (shard), both
// directions; tensor-core path only
cudaError_t launch_shard_states(const Problem &p, cudaStream_t stream);

// cached block decode on the tensor cores (bf16, headdim 64, d_state 128,
// blocks of at most 64 tokens): per batch row, the pool slot of its state and
// conv tail (null: row s uses slot s) and whether it commits (null: every row
// commits when state_out is given)
struct DecodeProblem {
    bimamba_dims dims;            // batch = rows, len = block length
    const void *xbc, *dt;
    const float *A, *D, *conv_w, *conv_b;
    const float *state;           // (pool, H, P, N)
    const void *tail;             // (pool, 4, ch)
    const int *slots;             // (batch) or null
    int pool;                     // pool size: slots must lie in [0, pool)
    const int *commit;            // (batch) or null
    float *state_out;             // (pool, H, P, N) or null; may alias state
    void *y;
    void *workspace;
    int *status;
};
bool decode_tc_supported(const bimamba_dims &d);
size_t decode_tc_workspace_bytes(const bimamba_dims &d);
cudaError_t launch_decode_tc(const DecodeProblem &q, cudaStream_t stream);
// the new conv tails of committed rows, in place in the pool: tail_pool[slot]
// <- last 4 raw tokens of (tail_pool[slot], block)
cudaError_t launch_tail_commit_pool(const void *block, void *tail_pool, const int *slots,
                                    const int *commit, int pool_size, int rows, int len, int ch,
                                    int *status, cudaStream_t stream);

// C = A . W^T on the tensor cores (bf16, fp32 accumulation), A (M, K) and W
// (N, K) row-major; columns [0, n_split) -> out0 (row stride n_split),
// columns [n_split, N) -> out1 (row stride N - n_split) as softplus(c + bias1)
struct GemmProblem {
    const void *a, *w;
    int M, N, K, n_split;
    void *out0, *out1;
    const float *bias1;
    int *status;
};
cudaError_t launch_gemm_tc(const GemmProblem &g, cudaStream_t stream);

// gradients of the mixer core (training path, fp32 results)
struct BackwardProblem {
    bimamba_dims dims;
    const void *xbc, *dt, *dy;
    const float *A, *D, *conv_w, *conv_b, *init;
    float *dxbc, *ddt, *dA, *dD, *dconv_w, *dconv_b, *dinit;
    void *workspace;
};
bool backward_supported(const bimamba_dims &d);
size_t backward_workspace_bytes(const bimamba_dims &d);
cudaError_t launch_backward(const BackwardProblem &q, cudaStream_t stream);

// the state and adjoint passes of the backward on the tensor cores (bf16,
// headdim 64, d_state 128): act = each stream's activated xBC, dact = its
// fp32 gradient (x part written, B/C parts added; zeroed by the caller),
// states = backward_tc_state_bytes of workspace
struct BackwardTcProblem {
    bimamba_dims dims;
    const void *act[2];
    const void *dt, *dy;
    const float *A, *D, *init;
    float *dact[2];
    float *ddt, *dA, *dD, *dinit;
    void *states;
};
bool backward_tc_supported(const bimamba_dims &d);
size_t backward_tc_state_bytes(const bimamba_dims &d);
cudaError_t launch_backward_tc(const BackwardTcProblem &q, cudaStream_t stream);

template <typename T>
cudaError_t launch_conv_silu(const void *u, void *out, const float *w, const float *bias,
                             const void *tail, int batch, int len, int ch, int rev, int silu,
                             cudaStream_t stream);

// both streams' conv + SiLU of one raw input with tied taps, in token order,
// and the conv backward of both streams, from TMA-staged tiles (raw rows,
// activations and gradients 16-byte aligned, ch a multiple of 8)
template <typename T>
cudaError_t launch_conv_silu_both_staged(const void *u, void *out_f, void *out_r, const float *w,
                                         const float *bias, int batch, int len, int ch, cudaStream_t stream);
// du = d(loss)/d(raw xBC) (fp32), dw / db += the tap and bias gradients
template <typename T>
cudaError_t launch_bwd_conv_staged(const void *u, const float *w, const float *bias, const float *dact_f,
                                   const float *dact_r, float *du, float *dw, float *db, int batch, int len,
                                   int ch, cudaStream_t stream);

template <typename T>
cudaError_t launch_scan_seq(const Problem &p, cudaStream_t stream);

template <typename T>
cudaError_t launch_tail_commit(const void *block, const void *tail, void *tail_out, int streams,
                               int len, int ch, cudaStream_t stream);

}  // namespace bimamba
