// api.cu -- host side of the C ABI declared in include/hstu_attn.h: argument validation,
// workspace sizing, the time-bucket threshold table, and the launch sequence on the
// caller's stream.  Allocates nothing and never synchronises in fwd/bwd.
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hstu {

namespace {

constexpr size_t kHeaderBytes = 256;   // status word, work-unit counter, padding

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

bool aligned16(const void *ptr) { return ((uintptr_t)ptr & 15u) == 0; }

// The bucket of |dt| decided in fp64 as floor(log((double)|dt| + 1.0) / div), unclamped.
double fp64_bucket(uint64_t a, double div) { return std::floor(std::log((double)a + 1.0) / div); }

// Smallest |dt| whose fp64 bucket is >= k (UINT64_MAX if none); the fp64 bucket is
// non-decreasing in |dt|, so a binary search over uint64 finds the boundary.
uint64_t threshold_for(int k, double div)
{
    if (fp64_bucket(UINT64_MAX, div) < (double)k) return UINT64_MAX;
    uint64_t lo = 0, hi = UINT64_MAX;   // invariant: bucket(hi) >= k
    while (lo < hi) {
        uint64_t mid = lo + (hi - lo) / 2;
        if (fp64_bucket(mid, div) >= (double)k) hi = mid; else lo = mid + 1;
    }
    return lo;
}

struct ThrEntry {
    std::vector<uint64_t> thr;
    int n_reach;
};

std::mutex g_thr_mu;
std::map<std::pair<double, int>, ThrEntry> g_thr_cache;

const ThrEntry &thresholds(double div, int nb)
{
    std::lock_guard<std::mutex> lock(g_thr_mu);
    auto key = std::make_pair(div, nb);
    auto it = g_thr_cache.find(key);
    if (it != g_thr_cache.end()) return it->second;
    ThrEntry e;
    e.n_reach = 0;
    for (int k = 1; k < nb; ++k) {
        uint64_t t = threshold_for(k, div);
        e.thr.push_back(t);
        if (t != UINT64_MAX) e.n_reach = k;
    }
    return g_thr_cache.emplace(key, std::move(e)).first->second;
}

hstu_status_t validate(const hstu_attn_params_t *p)
{
    if (!p) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->flags & ~(HSTU_FLAG_CTX_SEES_HISTORY | HSTU_FLAG_REL_ABS | HSTU_FLAG_CANDIDATES_ONLY))
        return HSTU_ERR_INVALID_ARGUMENT;
    if (p->batch < 0 || p->num_heads < 1 || p->total_tokens < 0) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->max_seqlen < 1) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->d_qk < 1 || p->d_v < 1 || p->d_qk > 256 || p->d_v > 256)
        return HSTU_ERR_INVALID_ARGUMENT;
    if ((int64_t)p->num_heads * p->d_v > 2048) return HSTU_ERR_UNSUPPORTED;
    if (p->rel_bias_len < 0 || p->time_bias_len < 0) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->time_bias_len > kMaxTimeBuckets) return HSTU_ERR_UNSUPPORTED;
    if (p->time_bias_len > 0 && !(p->time_bucket_div > 0.0 && std::isfinite(p->time_bucket_div)))
        return HSTU_ERR_INVALID_ARGUMENT;
    if (!std::isfinite(p->alpha) || !(p->ln_eps >= 0.f) || !std::isfinite(p->ln_eps))
        return HSTU_ERR_INVALID_ARGUMENT;
    if (p->dtype != HSTU_F32 && p->dtype != HSTU_BF16) return HSTU_ERR_INVALID_ARGUMENT;
    if ((int64_t)p->batch > 65535 || p->num_heads > 65535) return HSTU_ERR_UNSUPPORTED;
    if (p->total_tokens > ((int64_t)1 << 40)) return HSTU_ERR_UNSUPPORTED;
    return HSTU_OK;
}

// Test hook state (hstu_attn_set_wait_test): the pipeline-wait limit and the stall switch.
long long g_wait_limit = sm100::kWaitLimitCycles;
int32_t g_stall_test = 0;

DevParams make_dev_params(const hstu_attn_params_t *p, const int64_t *offsets, const int32_t *ctx,
                          const int32_t *tgt, const int64_t *ts, const float *rel,
                          const float *tb, void *workspace)
{
    DevParams d;
    std::memset(&d, 0, sizeof(d));
    d.B = p->batch;
    d.H = p->num_heads;
    d.dqk = p->d_qk;
    d.dv = p->d_v;
    d.N = p->max_seqlen;
    d.W = p->max_attn_len;
    d.T = p->total_tokens;
    d.D = p->num_heads * p->d_v;
    d.alpha = p->alpha;
    d.inv_N = 1.0f / (float)p->max_seqlen;
    d.eps = p->ln_eps;
    d.R = p->rel_bias_len;
    d.NB = p->time_bias_len;
    d.offsets = offsets;
    d.ctx = ctx;
    d.tgt = tgt;
    d.ts = ts;
    d.rel = rel;
    d.tb = tb;
    d.status = reinterpret_cast<int32_t *>(workspace);
    d.flags = p->flags;
    d.wait_limit = g_wait_limit;
    d.stall_test = g_stall_test;
    if (d.NB > 0) {
        const ThrEntry &e = thresholds(p->time_bucket_div, d.NB);
        d.n_thr = e.n_reach;
        for (int x = 0; x < d.NB - 1; ++x) d.thr[x] = e.thr[x];
    }
    return d;
}

size_t fwd_ws_bytes(const hstu_attn_params_t *p, bool need_y)
{
    size_t n = kHeaderBytes;
    if (need_y) n += align_up((size_t)p->total_tokens * p->num_heads * p->d_v * 4, 256);
    return n;
}

size_t bwd_ws_bytes(const hstu_attn_params_t *p)
{
    size_t n = kHeaderBytes;
    n += align_up((size_t)p->total_tokens * p->num_heads * p->d_v * 4, 256);     // dY
    if (p->dtype != HSTU_F32) {
        n += align_up((size_t)p->total_tokens * p->num_heads * p->d_qk * 4, 256);  // dQ fp32
        n += (size_t)kBwdMaxCtas * kMaxTimeBuckets * 4;   // per-CTA time-gradient rows
    }
    return n;
}

cudaEvent_t g_stage_ev[HSTU_NUM_STAGES][2];

// Records an event on s.  Inside a stream capture the record becomes a graph node of its
// own (external), so that each replay of the graph stamps the event.
void record_stage_event(cudaEvent_t e, cudaStream_t s)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(e, s, cudaEventRecordExternal);
    else
        cudaEventRecord(e, s);
}

struct StageScope {
    int stage;
    cudaStream_t s;
    StageScope(int st, cudaStream_t str) : stage(st), s(str)
    {
        if (g_stage_ev[stage][0]) record_stage_event(g_stage_ev[stage][0], s);
    }
    ~StageScope()
    {
        if (g_stage_ev[stage][1]) record_stage_event(g_stage_ev[stage][1], s);
    }
};

#define HSTU_CUDA_TRY(expr)                                   \
    do {                                                      \
        cudaError_t err_ = (expr);                            \
        if (err_ != cudaSuccess) return HSTU_ERR_CUDA;        \
    } while (0)

}  // namespace

}  // namespace hstu

using namespace hstu;

extern "C" {

const char *hstu_status_string(hstu_status_t s)
{
    switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARGUMENT: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported configuration";
    case HSTU_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_DEVICE_DATA: return "invalid device data (see status bits)";
    }
    return "unknown status";
}

int32_t hstu_attn_version(void) { return 100; }

hstu_status_t hstu_attn_time_thresholds(double div, int32_t nb, uint64_t *out)
{
    if (!out || nb < 1 || nb > kMaxTimeBuckets || !(div > 0.0) || !std::isfinite(div))
        return HSTU_ERR_INVALID_ARGUMENT;
    const ThrEntry &e = thresholds(div, nb);
    for (int k = 0; k < nb - 1; ++k) out[k] = e.thr[k];
    return HSTU_OK;
}

hstu_status_t hstu_attn_set_wait_test(int64_t limit_cycles, int32_t stall)
{
    if (limit_cycles < 0 || (stall != 0 && stall != 1)) return HSTU_ERR_INVALID_ARGUMENT;
    g_wait_limit = limit_cycles == 0 ? sm100::kWaitLimitCycles : (long long)limit_cycles;
    g_stall_test = stall;
    return HSTU_OK;
}

hstu_status_t hstu_attn_set_stage_events(int32_t stage, void *start_event, void *stop_event)
{
    if (stage < 0 || stage >= HSTU_NUM_STAGES) return HSTU_ERR_INVALID_ARGUMENT;
    g_stage_ev[stage][0] = reinterpret_cast<cudaEvent_t>(start_event);
    g_stage_ev[stage][1] = reinterpret_cast<cudaEvent_t>(stop_event);
    return HSTU_OK;
}

hstu_status_t hstu_attn_fwd_workspace_size(const hstu_attn_params_t *p, size_t *bytes)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    if (!bytes) return HSTU_ERR_INVALID_ARGUMENT;
    *bytes = fwd_ws_bytes(p, true);
    return HSTU_OK;
}

hstu_status_t hstu_attn_bwd_workspace_size(const hstu_attn_params_t *p, size_t *bytes)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    if (!bytes) return HSTU_ERR_INVALID_ARGUMENT;
    *bytes = bwd_ws_bytes(p);
    return HSTU_OK;
}

hstu_status_t hstu_attn_fwd(const hstu_attn_params_t *p, const void *q, const void *k,
                            const void *v, const void *u, const int64_t *seq_offsets,
                            const int32_t *num_contextuals, const int32_t *num_targets,
                            const int64_t *timestamps, const float *rel_bias,
                            const float *time_bias, void *out, float *saved_y,
                            float *saved_mean, float *saved_rstd, void *workspace,
                            size_t workspace_bytes, void *stream)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    const bool train = saved_y != nullptr;
    if (train != (saved_mean != nullptr) || train != (saved_rstd != nullptr))
        return HSTU_ERR_INVALID_ARGUMENT;
    if (train && (p->flags & HSTU_FLAG_CANDIDATES_ONLY)) return HSTU_ERR_UNSUPPORTED;
    if (!workspace || !seq_offsets) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->total_tokens > 0 && (!q || !k || !v || !u || !out)) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->rel_bias_len > 0 && !rel_bias) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->time_bias_len > 0 && (!time_bias || !timestamps)) return HSTU_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {q, k, v, u, out, saved_y, workspace};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return HSTU_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < fwd_ws_bytes(p, !train)) return HSTU_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DevParams d = make_dev_params(p, seq_offsets, num_contextuals, num_targets, timestamps,
                                  rel_bias, time_bias, workspace);
    // status word (bytes 0-3) and the work-unit counter (bytes 8-15) of the header
    HSTU_CUDA_TRY(cudaMemsetAsync(workspace, 0, 16, s));
    if (p->batch == 0 || p->total_tokens == 0) return HSTU_OK;
    float *y = train ? saved_y
                     : reinterpret_cast<float *>(reinterpret_cast<char *>(workspace) + kHeaderBytes);
    {
        StageScope scope(HSTU_STAGE_FWD_ATTN, s);
        if (p->dtype == HSTU_F32)
            HSTU_CUDA_TRY(launch_simt_fwd<float>(d, q, k, v, y, s));
        else if (tc_fwd_supported(p->d_qk, p->d_v, p->total_tokens))
            HSTU_CUDA_TRY(launch_tc_fwd(
                d, q, k, v, y,
                reinterpret_cast<unsigned long long *>(reinterpret_cast<char *>(workspace) + 8),
                train, s));
        else
            HSTU_CUDA_TRY(launch_simt_fwd<__nv_bfloat16>(d, q, k, v, y, s));
    }
    {
        StageScope scope(HSTU_STAGE_FWD_NORM, s);
        if (p->dtype == HSTU_F32)
            HSTU_CUDA_TRY(launch_ln_gate<float>(d, y, u, out, saved_mean, saved_rstd, s));
        else
            HSTU_CUDA_TRY(launch_ln_gate<__nv_bfloat16>(d, y, u, out, saved_mean, saved_rstd, s));
    }
    return HSTU_OK;
}

hstu_status_t hstu_attn_bwd(const hstu_attn_params_t *p, const void *dout, const void *q,
                            const void *k, const void *v, const void *u,
                            const int64_t *seq_offsets, const int32_t *num_contextuals,
                            const int32_t *num_targets, const int64_t *timestamps,
                            const float *rel_bias, const float *time_bias, const float *saved_y,
                            const float *saved_mean, const float *saved_rstd, void *dq, void *dk,
                            void *dv, void *du, float *d_rel_bias, float *d_time_bias,
                            void *workspace, size_t workspace_bytes, void *stream)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    if (p->flags & HSTU_FLAG_CANDIDATES_ONLY) return HSTU_ERR_UNSUPPORTED;   // forward only
    if (!workspace || !seq_offsets) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->total_tokens > 0 &&
        (!dout || !q || !k || !v || !u || !saved_y || !saved_mean || !saved_rstd || !dq || !dk ||
         !dv || !du))
        return HSTU_ERR_INVALID_ARGUMENT;
    if (p->rel_bias_len > 0 && (!rel_bias || !d_rel_bias)) return HSTU_ERR_INVALID_ARGUMENT;
    if (p->time_bias_len > 0 && (!time_bias || !timestamps || !d_time_bias))
        return HSTU_ERR_INVALID_ARGUMENT;
    const void *ptrs[] = {dout, q, k, v, u, saved_y, dq, dk, dv, du, workspace};
    for (const void *x : ptrs)
        if (x && !aligned16(x)) return HSTU_ERR_INVALID_ARGUMENT;
    if (workspace_bytes < bwd_ws_bytes(p)) return HSTU_ERR_WORKSPACE_TOO_SMALL;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    DevParams d = make_dev_params(p, seq_offsets, num_contextuals, num_targets, timestamps,
                                  rel_bias, time_bias, workspace);
    // status word (bytes 0-3) and the work-unit counter (bytes 8-15) of the header
    HSTU_CUDA_TRY(cudaMemsetAsync(workspace, 0, 16, s));
    if (p->batch == 0 || p->total_tokens == 0) {
        if (p->rel_bias_len > 0)
            HSTU_CUDA_TRY(cudaMemsetAsync(d_rel_bias, 0, sizeof(float) * p->rel_bias_len, s));
        if (p->time_bias_len > 0)
            HSTU_CUDA_TRY(cudaMemsetAsync(d_time_bias, 0, sizeof(float) * p->time_bias_len, s));
        return HSTU_OK;
    }

    char *ws = reinterpret_cast<char *>(workspace) + kHeaderBytes;
    float *dy = reinterpret_cast<float *>(ws);
    ws += align_up((size_t)p->total_tokens * p->num_heads * p->d_v * 4, 256);
    const int64_t nq = p->total_tokens * p->num_heads * p->d_qk;
    const bool f32 = p->dtype == HSTU_F32;
    const bool tc = !f32 && tc_bwd_supported(p->d_qk, p->d_v, p->total_tokens);
    float *dq_acc = f32 ? reinterpret_cast<float *>(dq) : reinterpret_cast<float *>(ws);
    float *tb_slots = f32 ? nullptr
                          : reinterpret_cast<float *>(ws + align_up((size_t)nq * 4, 256));
    // the LayerNorm backward zeroes the dQ accumulator and the table gradients on its way
    BwdZero zero;
    zero.rows = dq_acc;
    zero.row_floats = (int64_t)p->num_heads * p->d_qk;
    zero.a = d_rel_bias;
    zero.na = p->rel_bias_len;
    zero.b = d_time_bias;
    zero.nb = p->time_bias_len;
    {
        StageScope scope(HSTU_STAGE_BWD_NORM, s);
        if (f32)
            HSTU_CUDA_TRY(launch_ln_gate_bwd<float>(d, dout, u, saved_y, saved_mean, saved_rstd,
                                                    du, dy, false, zero, s));
        else
            HSTU_CUDA_TRY(launch_ln_gate_bwd<__nv_bfloat16>(d, dout, u, saved_y, saved_mean,
                                                            saved_rstd, du, dy, tc, zero, s));
    }
    {
        StageScope scope(HSTU_STAGE_BWD_ATTN, s);
        if (f32) {
            HSTU_CUDA_TRY(launch_simt_bwd<float>(d, q, k, v, dy, dq_acc, dk, dv, d_rel_bias,
                                                 d_time_bias, s));
        } else if (tc) {
            HSTU_CUDA_TRY(launch_tc_bwd(
                d, q, k, v, dy, dq_acc, dk, dv, d_rel_bias, d_time_bias, tb_slots,
                reinterpret_cast<unsigned long long *>(reinterpret_cast<char *>(workspace) + 8),
                s));
            HSTU_CUDA_TRY(launch_convert<__nv_bfloat16>(dq_acc, dq, nq, s));
        } else {
            HSTU_CUDA_TRY(launch_simt_bwd<__nv_bfloat16>(d, q, k, v, dy, dq_acc, dk, dv,
                                                         d_rel_bias, d_time_bias, s));
            HSTU_CUDA_TRY(launch_convert<__nv_bfloat16>(dq_acc, dq, nq, s));
        }
    }
    return HSTU_OK;
}

hstu_status_t hstu_attn_read_device_status(const void *workspace, void *stream, int32_t *code)
{
    if (!workspace || !code) return HSTU_ERR_INVALID_ARGUMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t h = 0;
    if (cudaMemcpyAsync(&h, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return HSTU_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
    *code = h;
    return h ? HSTU_ERR_DEVICE_DATA : HSTU_OK;
}

hstu_status_t hstu_attn_debug_mask(const hstu_attn_params_t *p, const int64_t *seq_offsets,
                                   const int32_t *num_contextuals, const int32_t *num_targets,
                                   int32_t seq, int32_t seq_len, uint32_t *bits, void *stream)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    if (!seq_offsets || !bits || seq < 0 || seq >= p->batch || seq_len < 0)
        return HSTU_ERR_INVALID_ARGUMENT;
    if (seq_len == 0) return HSTU_OK;
    DevParams d = make_dev_params(p, seq_offsets, num_contextuals, num_targets, nullptr, nullptr,
                                  nullptr, nullptr);
    HSTU_CUDA_TRY(launch_debug_mask(d, seq, seq_len, bits, reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_attn_debug_kernel_mask(const hstu_attn_params_t *p,
                                          const int64_t *seq_offsets,
                                          const int32_t *num_contextuals,
                                          const int32_t *num_targets, int32_t seq,
                                          int32_t kernel, int32_t row_begin, int32_t row_count,
                                          int32_t key_count, uint32_t *bits, void *stream)
{
    hstu_status_t st = validate(p);
    if (st != HSTU_OK) return st;
    if (!seq_offsets || !bits || seq < 0 || seq >= p->batch || (kernel != 0 && kernel != 1) ||
        row_begin < 0 || row_count < 0 || key_count < 0 || key_count % 32 != 0)
        return HSTU_ERR_INVALID_ARGUMENT;
    if (row_count == 0 || key_count == 0) return HSTU_OK;
    DevParams d = make_dev_params(p, seq_offsets, num_contextuals, num_targets, nullptr, nullptr,
                                  nullptr, nullptr);
    HSTU_CUDA_TRY(launch_debug_kernel_mask(d, seq, kernel, row_begin, row_count, key_count, bits,
                                           reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_layer_norm_rows(const void *x, void *y, int64_t rows, int32_t width,
                                   float eps, void *stream)
{
    if (rows < 0 || width < 32 || width > 1024 || width % 32 != 0 || !(eps >= 0.f) ||
        (rows > 0 && (!x || !y)))
        return HSTU_ERR_INVALID_ARGUMENT;
    HSTU_CUDA_TRY(launch_ln_rows(x, y, rows, width, eps, reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_uvqk_proj(const void *x, const void *w, const float *bias, int64_t tokens,
                             int32_t d_model, int32_t num_heads, int32_t d_qk, int32_t d_v,
                             int32_t silu, void *u, void *v, void *q, void *k, int32_t *status,
                             void *stream)
{
    if (tokens < 0 || tokens > INT32_MAX || d_model < 64 || d_model % 64 != 0 || num_heads < 1 ||
        d_qk < 1 || d_v < 1 || ((int64_t)num_heads * d_qk) % 64 != 0 ||
        ((int64_t)num_heads * d_v) % 64 != 0 || (silu != 0 && silu != 1))
        return HSTU_ERR_INVALID_ARGUMENT;
    const int64_t N = 2 * (int64_t)num_heads * (d_v + d_qk);
    if (N > 65536) return HSTU_ERR_UNSUPPORTED;
    if (tokens == 0) return HSTU_OK;
    const void *ptrs[] = {x, w, bias, u, v, q, k};
    for (int x_ = 0; x_ < 7; ++x_)
        if ((x_ != 2 && !ptrs[x_]) || !aligned16(ptrs[x_])) return HSTU_ERR_INVALID_ARGUMENT;
    const int hv = num_heads * d_v, hq = num_heads * d_qk;
    const int lo[5] = {0, hv, 2 * hv, 2 * hv + hq, 2 * hv + 2 * hq};
    void *outs[4] = {u, v, q, k};
    HSTU_CUDA_TRY(launch_gemm(x, w, (int)tokens, (int)N, d_model, bias, silu != 0, nullptr, 4, lo,
                              outs, status, g_wait_limit, reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_out_proj(const void *z, const void *w_o, const float *bias, const void *x,
                            int64_t tokens, int32_t d_in, int32_t d_model, void *out,
                            int32_t *status, void *stream)
{
    if (tokens < 0 || tokens > INT32_MAX || d_in < 64 || d_in % 64 != 0 || d_model < 64 ||
        d_model % 64 != 0 || d_model > 65536)
        return HSTU_ERR_INVALID_ARGUMENT;
    if (tokens == 0) return HSTU_OK;
    const void *ptrs[] = {z, w_o, bias, x, out};
    for (int x_ = 0; x_ < 5; ++x_)
        if (((x_ == 0 || x_ == 1 || x_ == 4) && !ptrs[x_]) || !aligned16(ptrs[x_]))
            return HSTU_ERR_INVALID_ARGUMENT;
    const int lo[2] = {0, d_model};
    void *outs[1] = {out};
    HSTU_CUDA_TRY(launch_gemm(z, w_o, (int)tokens, d_model, d_in, bias, false, x, 1, lo, outs,
                              status, g_wait_limit, reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_stochastic_length(const int64_t *seq_offsets, const int32_t *num_contextuals,
                                     const int32_t *num_targets, int32_t batch,
                                     int64_t total_tokens, const float *keys, int32_t budget,
                                     int64_t *out_rows, int64_t *out_offsets, int32_t *status,
                                     void *stream)
{
    if (batch < 0 || batch > 65535 || total_tokens < 0 || budget < 0 || !seq_offsets ||
        !out_offsets || (total_tokens > 0 && (!keys || !out_rows)))
        return HSTU_ERR_INVALID_ARGUMENT;
    DevParams d;
    std::memset(&d, 0, sizeof(d));
    d.B = batch;
    d.T = total_tokens;
    d.N = INT32_MAX;          // no length limit here
    d.offsets = seq_offsets;
    d.ctx = num_contextuals;
    d.tgt = num_targets;
    d.status = status;
    HSTU_CUDA_TRY(launch_stochastic_length(d, keys, budget, out_rows, out_offsets,
                                           reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_gather_rows(const void *src, int64_t row_bytes, const int64_t *rows,
                               const int64_t *n_rows, int64_t max_rows, void *dst, void *stream)
{
    if (row_bytes <= 0 || max_rows < 0 || !n_rows || (max_rows > 0 && (!src || !rows || !dst)))
        return HSTU_ERR_INVALID_ARGUMENT;
    HSTU_CUDA_TRY(launch_gather_rows(src, row_bytes, rows, n_rows, max_rows, dst,
                                     reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

hstu_status_t hstu_jagged_concat(int32_t n_parts, const void *const *values,
                                 const int64_t *const *offsets, int32_t batch, int64_t row_bytes,
                                 void *out_values, int64_t *out_offsets, void *stream)
{
    if (n_parts < 1 || n_parts > kMaxConcatParts || batch < 0 || row_bytes <= 0 || !values ||
        !offsets || !out_values || !out_offsets)
        return HSTU_ERR_INVALID_ARGUMENT;
    for (int q = 0; q < n_parts; ++q)
        if (!values[q] || !offsets[q]) return HSTU_ERR_INVALID_ARGUMENT;
    HSTU_CUDA_TRY(launch_jagged_concat(n_parts, values, offsets, batch, row_bytes, out_values,
                                       out_offsets, reinterpret_cast<cudaStream_t>(stream)));
    return HSTU_OK;
}

}  // extern "C"
