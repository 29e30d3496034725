// api.cu -- host side of the C ABI declared in include/bimamba.h: argument
// validation (nothing is launched when it fails), workspace sizing, the
// per-device status word, and dispatch to the sm_100a kernels.
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "dispatch.h"

namespace bimamba {

__device__ int g_status;

static std::atomic<unsigned long long> g_launches{0};

void count_launch(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

static thread_local TimingEvents t_events{nullptr, nullptr};

TimingEvents timing_events() { return t_events; }

int *device_status_word()
{
    // one address per device; resolved with that device current
    static std::mutex mu;
    static int *addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        addr[dev] = static_cast<int *>(p);
    }
    return addr[dev];
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static bool pow2_in(int v, int lo, int hi)
{
    return v >= lo && v <= hi && (v & (v - 1)) == 0;
}

// Shape/dtype checks common to every entry point; returns BIMAMBA_OK or an error.
static int check_dims(const bimamba_dims *d)
{
    if (!d) return BIMAMBA_ERR_INVALID;
    if (d->batch < 0 || d->len < 0 || d->heads <= 0 || d->headdim <= 0 || d->d_state <= 0 ||
        d->ngroups <= 0 || d->d_conv <= 0)
        return BIMAMBA_ERR_INVALID;
    if (d->dtype != BIMAMBA_F32 && d->dtype != BIMAMBA_BF16) return BIMAMBA_ERR_INVALID;
    if (d->heads % d->ngroups != 0) return BIMAMBA_ERR_INVALID;
    if (d->ngroups != 1 || d->d_conv != 4) return BIMAMBA_ERR_UNSUPPORTED;
    if (d->headdim % 8 != 0 || d->headdim > 128) return BIMAMBA_ERR_UNSUPPORTED;
    if (!pow2_in(d->d_state, 8, 256)) return BIMAMBA_ERR_UNSUPPORTED;
    // sizes must fit the kernels' 32-bit token indexing and 64-bit offsets
    const int64_t ch = (int64_t)d->heads * d->headdim + 2LL * d->ngroups * d->d_state;
    if (ch > (1 << 20) || (int64_t)d->batch * d->len > (int64_t)1 << 40) return BIMAMBA_ERR_UNSUPPORTED;
    if ((int64_t)d->batch > 65535 || d->heads > 65535) return BIMAMBA_ERR_UNSUPPORTED;
    return BIMAMBA_OK;
}

static int cuda_status(cudaError_t e) { return e == cudaSuccess ? BIMAMBA_OK : BIMAMBA_ERR_CUDA; }

int check_block_decode(const bimamba_dims *d, const void *xbc_block, const void *dt_block,
                       const float *A, const float *D, const float *conv_w, const float *conv_b,
                       const float *state, const void *tail, const void *y, const float *state_out,
                       const void *tail_out)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    if (d->batch == 0) return BIMAMBA_OK;
    if (d->len == 0) return BIMAMBA_ERR_INVALID;
    if (!xbc_block || !dt_block || !A || !D || !conv_w || !state || !tail || !y)
        return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y, state_out, tail_out};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    const size_t esz = d->dtype == BIMAMBA_F32 ? 4 : 2;
    const int ch = d->heads * d->headdim + 2 * d->ngroups * d->d_state;
    const size_t tail_bytes = (size_t)d->batch * 4 * ch * esz;
    if (tail_out) {
        const char *a = static_cast<const char *>(tail), *b = static_cast<const char *>(tail_out);
        if (a < b + tail_bytes && b < a + tail_bytes) return BIMAMBA_ERR_INVALID;
    }
    return BIMAMBA_OK;
}

}  // namespace bimamba

using namespace bimamba;

extern "C" {

int bimamba_version(void) { return (1 << 16) | 0; }

unsigned long long bimamba_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int bimamba_set_timing_events(void *start, void *stop)
{
    if ((start == nullptr) != (stop == nullptr)) return BIMAMBA_ERR_INVALID;
    t_events.start = static_cast<cudaEvent_t>(start);
    t_events.stop = static_cast<cudaEvent_t>(stop);
    return BIMAMBA_OK;
}

const char *bimamba_strerror(int status)
{
    switch (status) {
    case BIMAMBA_OK: return "ok";
    case BIMAMBA_ERR_INVALID: return "invalid argument";
    case BIMAMBA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case BIMAMBA_ERR_CUDA: return "CUDA runtime error";
    case BIMAMBA_ERR_TIMEOUT: return "a kernel's bounded wait timed out";
    case BIMAMBA_ERR_WORKSPACE: return "workspace missing or too small";
    default: return "unknown status";
    }
}

int bimamba_get_error(bimamba_stream_t stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    int *w = device_status_word();
    if (!w) return BIMAMBA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return BIMAMBA_ERR_CUDA;
    if (v) {
        const int zero = 0;
        if (cudaMemcpy(w, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
            return BIMAMBA_ERR_CUDA;
    }
    if (v & kStatusTimeout) return BIMAMBA_ERR_TIMEOUT;
    if (v & kStatusBadSlot) return BIMAMBA_ERR_INVALID;
    return BIMAMBA_OK;
}

int bimamba_conv_silu(const void *u, void *out, const float *w, const float *bias,
                      const void *tail, int batch, int len, int ch, int d_conv, int reverse,
                      int silu, int dtype, bimamba_stream_t stream)
{
    if (batch < 0 || len < 0 || ch <= 0) return BIMAMBA_ERR_INVALID;
    if (dtype != BIMAMBA_F32 && dtype != BIMAMBA_BF16) return BIMAMBA_ERR_INVALID;
    if (d_conv != 4 || ch % 8 != 0) return BIMAMBA_ERR_UNSUPPORTED;
    if (batch > 65535 || (len + 63) / 64 > 65535) return BIMAMBA_ERR_UNSUPPORTED;
    if (batch == 0 || len == 0) return BIMAMBA_OK;
    if (!u || !out || !w) return BIMAMBA_ERR_INVALID;
    if (reverse && tail) return BIMAMBA_ERR_INVALID;
    if (!aligned16(u) || !aligned16(out) || !aligned16(w) || (tail && !aligned16(tail)))
        return BIMAMBA_ERR_INVALID;
    const size_t esz = dtype == BIMAMBA_F32 ? 4 : 2;
    const char *ub = static_cast<const char *>(u), *ob = static_cast<const char *>(out);
    const size_t bytes = (size_t)batch * len * ch * esz;
    if (ub < ob + bytes && ob < ub + bytes) return BIMAMBA_ERR_INVALID;  // overlap
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = dtype == BIMAMBA_F32
                        ? launch_conv_silu<float>(u, out, w, bias, tail, batch, len, ch, reverse, silu, s)
                        : launch_conv_silu<__nv_bfloat16>(u, out, w, bias, tail, batch, len, ch,
                                                          reverse, silu, s);
    return cuda_status(e);
}

size_t bimamba_workspace_bytes(const bimamba_dims *d)
{
    if (check_dims(d) != BIMAMBA_OK) return 0;
    return workspace_bytes_for(*d);
}

int bimamba_launch_plan(const bimamba_dims *d, int *out)
{
    if (!out) return BIMAMBA_ERR_INVALID;
    const int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    out[0] = tc_path_supported(*d) ? 1 : 0;
    if (out[0]) {
        tc_launch_plan(*d, out + 1);
    } else {
        out[1] = 1;
        out[2] = (d->len + 127) / 128;
        out[3] = 0;
    }
    return BIMAMBA_OK;
}

// Shared by the full scan (tied or untied) and the cached block decode.
// Index 0 of each pair is the forward stream's input, index 1 the reverse's.
static int run_bimamba(const bimamba_dims *d, const void *const xbc[2], const void *const dt[2],
                       const float *const A[2], const float *const D[2],
                       const float *const conv_w[2], const float *const conv_b[2], int concat,
                       const void *tail, const float *init, float *fin, void *y,
                       void *workspace, size_t workspace_bytes, cudaStream_t s)
{
    const size_t need = workspace_bytes_for(*d);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
        return BIMAMBA_ERR_WORKSPACE;
    Problem pr{};
    pr.dims = *d;
    for (int i = 0; i < 2; ++i) {
        pr.xbc[i] = xbc[i]; pr.dt[i] = dt[i]; pr.A[i] = A[i]; pr.D[i] = D[i];
        pr.conv_w[i] = conv_w[i]; pr.conv_b[i] = conv_b[i];
    }
    pr.concat = concat;
    pr.tail = tail;
    pr.init = init; pr.fin = fin; pr.y = y;
    pr.workspace = workspace; pr.workspace_bytes = workspace_bytes;
    pr.status = device_status_word();
    return cuda_status(launch_bimamba(pr, s));
}

static int run_tied(const bimamba_dims *d, const void *xbc, const void *dt, const float *A,
                    const float *D, const float *conv_w, const float *conv_b, const void *tail,
                    const float *init, float *fin, void *y, void *workspace,
                    size_t workspace_bytes, cudaStream_t s)
{
    const void *x2[2] = {xbc, xbc}, *dt2[2] = {dt, dt};
    const float *A2[2] = {A, A}, *D2[2] = {D, D}, *w2[2] = {conv_w, conv_w}, *b2[2] = {conv_b, conv_b};
    return run_bimamba(d, x2, dt2, A2, D2, w2, b2, 0, tail, init, fin, y, workspace,
                       workspace_bytes, s);
}

// Empty sequence: y is empty; the forward state passes through.
static int pass_state_through(const bimamba_dims *d, const float *init_state, float *final_state,
                              cudaStream_t s)
{
    const size_t state_bytes = sizeof(float) * (size_t)d->batch * d->heads * d->headdim * d->d_state;
    if (!final_state || init_state == final_state) return BIMAMBA_OK;
    cudaError_t e = init_state ? cudaMemcpyAsync(final_state, init_state, state_bytes,
                                                 cudaMemcpyDeviceToDevice, s)
                               : cudaMemsetAsync(final_state, 0, state_bytes, s);
    return cuda_status(e);
}

int bimamba_ssd_fwd_rev(const bimamba_dims *d, const void *xbc, const void *dt, const float *A,
                        const float *D, const float *conv_w, const float *conv_b,
                        const float *init_state, float *final_state, void *y, void *workspace,
                        size_t workspace_bytes, bimamba_stream_t stream)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d->batch == 0) return BIMAMBA_OK;
    if (d->len == 0) return pass_state_through(d, init_state, final_state, s);
    if (!xbc || !dt || !A || !D || !y) return BIMAMBA_ERR_INVALID;
    if (conv_b && !conv_w) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc, dt, A, D, y, conv_w, conv_b, init_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    return run_tied(d, xbc, dt, A, D, conv_w, conv_b, nullptr, init_state, final_state, y,
                    workspace, workspace_bytes, s);
}

int bimamba_ssd_fwd_rev_untied(const bimamba_dims *d, const void *xbc_f, const void *xbc_r,
                               const void *dt_f, const void *dt_r, const float *A_f,
                               const float *A_r, const float *D_f, const float *D_r,
                               const float *conv_w_f, const float *conv_w_r,
                               const float *conv_b_f, const float *conv_b_r,
                               const float *init_state, float *final_state, void *y, int fusion,
                               void *workspace, size_t workspace_bytes, bimamba_stream_t stream)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    if (fusion != BIMAMBA_FUSE_SUM && fusion != BIMAMBA_FUSE_CONCAT) return BIMAMBA_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d->batch == 0) return BIMAMBA_OK;
    if (d->len == 0) return pass_state_through(d, init_state, final_state, s);
    if (!xbc_f || !xbc_r || !dt_f || !dt_r || !A_f || !A_r || !D_f || !D_r || !y)
        return BIMAMBA_ERR_INVALID;
    if ((conv_b_f && !conv_w_f) || (conv_b_r && !conv_w_r)) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc_f, xbc_r, dt_f, dt_r, A_f, A_r, D_f, D_r, y, conv_w_f, conv_w_r,
                          conv_b_f, conv_b_r, init_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    const void *x2[2] = {xbc_f, xbc_r}, *dt2[2] = {dt_f, dt_r};
    const float *A2[2] = {A_f, A_r}, *D2[2] = {D_f, D_r};
    const float *w2[2] = {conv_w_f, conv_w_r}, *b2[2] = {conv_b_f, conv_b_r};
    return run_bimamba(d, x2, dt2, A2, D2, w2, b2, fusion == BIMAMBA_FUSE_CONCAT, nullptr,
                       init_state, final_state, y, workspace, workspace_bytes, s);
}

// Sequence shards: a shard's inputs, halos and tied parameters into a Problem.
static int shard_problem(const bimamba_dims *d, const void *xbc, const void *dt, const float *A,
                         const float *D, const float *conv_w, const float *conv_b,
                         const void *tail, const void *head, void *workspace,
                         size_t workspace_bytes, Problem &pr)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    if (!tc_path_supported(*d)) return BIMAMBA_ERR_UNSUPPORTED;
    if (!xbc || !dt || !A) return BIMAMBA_ERR_INVALID;
    if (conv_b && !conv_w) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc, dt, A, D, conv_w, conv_b, tail, head};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return BIMAMBA_ERR_INVALID;
    const size_t need = workspace_bytes_for(*d);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
        return BIMAMBA_ERR_WORKSPACE;
    pr = Problem{};
    pr.dims = *d;
    for (int i = 0; i < 2; ++i) {
        pr.xbc[i] = xbc; pr.dt[i] = dt; pr.A[i] = A; pr.D[i] = D;
        pr.conv_w[i] = conv_w; pr.conv_b[i] = conv_b;
    }
    pr.tail = tail;
    pr.head = head;
    pr.workspace = workspace;
    pr.workspace_bytes = workspace_bytes;
    pr.status = device_status_word();
    return BIMAMBA_OK;
}

int bimamba_shard_states(const bimamba_dims *d, const void *xbc, const void *dt, const float *A,
                         const float *conv_w, const float *conv_b, const void *tail,
                         const void *head, float *states, float *decays, void *workspace,
                         size_t workspace_bytes, bimamba_stream_t stream)
{
    Problem pr;
    int st = shard_problem(d, xbc, dt, A, nullptr, conv_w, conv_b, tail, head, workspace,
                           workspace_bytes, pr);
    if (st != BIMAMBA_OK) return st;
    if (!states || !decays || !aligned16(states) || !aligned16(decays)) return BIMAMBA_ERR_INVALID;
    if (d->batch == 0) return BIMAMBA_OK;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (d->len == 0) {
        // an empty shard leaves every state unchanged: zero states, zero log-decay
        const size_t ns = (size_t)2 * d->batch * d->heads * d->headdim * d->d_state;
        cudaError_t e = cudaMemsetAsync(states, 0, ns * sizeof(float), s);
        if (e == cudaSuccess)
            e = cudaMemsetAsync(decays, 0, (size_t)2 * d->batch * d->heads * sizeof(float), s);
        return cuda_status(e);
    }
    pr.states_out = states;
    pr.dec_out = decays;
    return cuda_status(launch_shard_states(pr, s));
}

int bimamba_ssd_fwd_rev_shard(const bimamba_dims *d, const void *xbc, const void *dt,
                              const float *A, const float *D, const float *conv_w,
                              const float *conv_b, const void *tail, const void *head,
                              const float *init_state, const float *all_states,
                              const float *all_decays, int rank, int nranks, float *final_state,
                              void *y, void *workspace, size_t workspace_bytes,
                              bimamba_stream_t stream)
{
    Problem pr;
    int st = shard_problem(d, xbc, dt, A, D, conv_w, conv_b, tail, head, workspace,
                           workspace_bytes, pr);
    if (st != BIMAMBA_OK) return st;
    if (!D || !y || nranks < 1 || rank < 0 || rank >= nranks) return BIMAMBA_ERR_INVALID;
    if (nranks > 1 && (!all_states || !all_decays)) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {init_state, all_states, all_decays, final_state, y};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return BIMAMBA_ERR_INVALID;
    if (d->batch == 0 || d->len == 0) return d->len == 0 && d->batch > 0 ? BIMAMBA_ERR_INVALID
                                                                       : BIMAMBA_OK;
    pr.init = init_state;
    pr.fin = final_state;
    pr.y = y;
    if (nranks > 1) {
        pr.shard_states = all_states;
        pr.shard_dec = all_decays;
    }
    pr.rank = rank;
    pr.nranks = nranks;
    return cuda_status(launch_bimamba(pr, reinterpret_cast<cudaStream_t>(stream)));
}

// The tensor-core decode kernels (blocks of at most 64 tokens): state and
// tail from pool slots, per-row commit.
static int run_decode_tc(const bimamba_dims *d, const void *xbc_block, const void *dt_block,
                         const float *A, const float *D, const float *conv_w, const float *conv_b,
                         const float *state, const void *tail, const int *slots, int pool,
                         const int *commit, float *state_out, void *y, void *workspace,
                         size_t workspace_bytes, cudaStream_t s)
{
    const size_t need = workspace_bytes_for(*d);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return BIMAMBA_ERR_WORKSPACE;
    DecodeProblem q{};
    q.dims = *d;
    q.xbc = xbc_block; q.dt = dt_block; q.A = A; q.D = D; q.conv_w = conv_w; q.conv_b = conv_b;
    q.state = state; q.tail = tail; q.slots = slots; q.pool = pool; q.commit = commit;
    q.state_out = state_out; q.y = y; q.workspace = workspace;
    q.status = device_status_word();
    return cuda_status(launch_decode_tc(q, s));
}

int bimamba_block_decode(const bimamba_dims *d, const void *xbc_block, const void *dt_block,
                         const float *A, const float *D, const float *conv_w,
                         const float *conv_b, const float *state, const void *tail, void *y,
                         float *state_out, void *tail_out, void *workspace,
                         size_t workspace_bytes, bimamba_stream_t stream)
{
    int st = check_block_decode(d, xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y,
                                state_out, tail_out);
    if (st != BIMAMBA_OK) return st;
    if (d->batch == 0) return BIMAMBA_OK;
    const int ch = d->heads * d->headdim + 2 * d->ngroups * d->d_state;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (decode_tc_supported(*d))
        st = run_decode_tc(d, xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, nullptr,
                           d->batch, nullptr, state_out, y, workspace, workspace_bytes, s);
    else
        st = run_tied(d, xbc_block, dt_block, A, D, conv_w, conv_b, tail, state, state_out, y,
                      workspace, workspace_bytes, s);
    if (st != BIMAMBA_OK || !tail_out) return st;
    cudaError_t e = d->dtype == BIMAMBA_F32
                        ? launch_tail_commit<float>(xbc_block, tail, tail_out, d->batch, d->len, ch, s)
                        : launch_tail_commit<__nv_bfloat16>(xbc_block, tail, tail_out, d->batch,
                                                            d->len, ch, s);
    return cuda_status(e);
}

int bimamba_block_decode_pool(const bimamba_dims *d, const void *xbc_block, const void *dt_block,
                              const float *A, const float *D, const float *conv_w,
                              const float *conv_b, float *state_pool, void *tail_pool,
                              int pool_size, const int *slots, const int *commit, void *y,
                              void *workspace, size_t workspace_bytes, bimamba_stream_t stream)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    if (d->batch == 0) return BIMAMBA_OK;
    if (!decode_tc_supported(*d)) return BIMAMBA_ERR_UNSUPPORTED;
    if (pool_size < 1 || !xbc_block || !dt_block || !A || !D || !conv_w || !state_pool ||
        !tail_pool || !slots || !y)
        return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc_block, dt_block, A, D, conv_w, conv_b, state_pool, tail_pool, y};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    const int ch = d->heads * d->headdim + 2 * d->ngroups * d->d_state;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    st = run_decode_tc(d, xbc_block, dt_block, A, D, conv_w, conv_b, state_pool, tail_pool, slots,
                       pool_size, commit, state_pool, y, workspace, workspace_bytes, s);
    if (st != BIMAMBA_OK) return st;
    return cuda_status(launch_tail_commit_pool(xbc_block, tail_pool, slots, commit, pool_size,
                                               d->batch, d->len, ch, device_status_word(), s));
}

int bimamba_in_proj(int tokens, int d_model, int heads, int headdim, int d_state, const void *u,
                    const void *w_in, const float *dt_bias, void *xbc, void *dt,
                    bimamba_stream_t stream)
{
    if (tokens < 0 || d_model <= 0 || heads <= 0 || headdim <= 0 || d_state <= 0)
        return BIMAMBA_ERR_INVALID;
    if (d_model % 8 != 0) return BIMAMBA_ERR_UNSUPPORTED;
    const long long ch = (long long)heads * headdim + 2LL * d_state;
    if (ch + heads > (1 << 20) || tokens > (1 << 30)) return BIMAMBA_ERR_UNSUPPORTED;
    if (tokens == 0) return BIMAMBA_OK;
    if (!u || !w_in || !xbc || !dt) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {u, w_in, dt_bias, xbc, dt};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    GemmProblem g{};
    g.a = u; g.w = w_in;
    g.M = tokens; g.N = (int)(ch + heads); g.K = d_model; g.n_split = (int)ch;
    g.out0 = xbc; g.out1 = dt; g.bias1 = dt_bias;
    g.status = device_status_word();
    return cuda_status(launch_gemm_tc(g, reinterpret_cast<cudaStream_t>(stream)));
}

int bimamba_out_proj(int tokens, int d_inner, int d_model, const void *y, const void *w_out,
                     void *out, bimamba_stream_t stream)
{
    if (tokens < 0 || d_inner <= 0 || d_model <= 0) return BIMAMBA_ERR_INVALID;
    if (d_inner % 8 != 0) return BIMAMBA_ERR_UNSUPPORTED;
    if (d_model > (1 << 20) || tokens > (1 << 30)) return BIMAMBA_ERR_UNSUPPORTED;
    if (tokens == 0) return BIMAMBA_OK;
    if (!y || !w_out || !out) return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {y, w_out, out};
    for (const void *p : ptrs)
        if (!aligned16(p)) return BIMAMBA_ERR_INVALID;
    GemmProblem g{};
    g.a = y; g.w = w_out;
    g.M = tokens; g.N = d_model; g.K = d_inner; g.n_split = d_model;
    g.out0 = out;
    g.status = device_status_word();
    return cuda_status(launch_gemm_tc(g, reinterpret_cast<cudaStream_t>(stream)));
}

size_t bimamba_backward_workspace_bytes(const bimamba_dims *d)
{
    if (check_dims(d) != BIMAMBA_OK || !backward_supported(*d)) return 0;
    return backward_workspace_bytes(*d);
}

int bimamba_ssd_fwd_rev_backward(const bimamba_dims *d, const void *xbc, const void *dt,
                                 const float *A, const float *D, const float *conv_w,
                                 const float *conv_b, const float *init_state, const void *dy,
                                 float *dxbc, float *ddt, float *dA, float *dD, float *dconv_w,
                                 float *dconv_b, float *dinit, void *workspace,
                                 size_t workspace_bytes, bimamba_stream_t stream)
{
    int st = check_dims(d);
    if (st != BIMAMBA_OK) return st;
    if (!backward_supported(*d)) return BIMAMBA_ERR_UNSUPPORTED;
    if (d->batch == 0 || d->len == 0) return BIMAMBA_ERR_INVALID;
    if (!xbc || !dt || !A || !D || !conv_w || !dy || !dxbc || !ddt || !dA || !dD || !dconv_w)
        return BIMAMBA_ERR_INVALID;
    const void *ptrs[] = {xbc, dt, A, D, conv_w, conv_b, init_state, dy, dxbc, ddt, dA, dD,
                          dconv_w, dconv_b, dinit};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BIMAMBA_ERR_INVALID;
    const size_t need = backward_workspace_bytes(*d);
    if (!workspace || workspace_bytes < need || !aligned16(workspace)) return BIMAMBA_ERR_WORKSPACE;
    BackwardProblem q{};
    q.dims = *d;
    q.xbc = xbc; q.dt = dt; q.dy = dy; q.A = A; q.D = D; q.conv_w = conv_w; q.conv_b = conv_b;
    q.init = init_state;
    q.dxbc = dxbc; q.ddt = ddt; q.dA = dA; q.dD = dD; q.dconv_w = dconv_w; q.dconv_b = dconv_b;
    q.dinit = dinit;
    q.workspace = workspace;
    return cuda_status(launch_backward(q, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
