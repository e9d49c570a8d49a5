// simt.cu -- CUDA-core kernels of jagged HSTU attention: the fp32 attention forward and
// backward (the precision path for fp32 inputs), the per-token LayerNorm + U gating, and
// the LayerNorm/gating backward.
//
// Forward per (sequence, head, 64-row query tile): for every 64-key tile that holds a
// valid pair, S = Q K^T in fp32, s = alpha*S + b, A = mask ? SiLU(s) : 0 (the mask is applied
// after the nonlinearity, as "HSTU tensor by tensor: SiLU aggregation, temporal bias and
// gating", section "Do not copy softmax masking mechanically", requires), Y += A V; at the end
// Y is scaled by 1/N ("HSTU-MUSA: HSTU for Moore Threads (MUSA)", "Accuracy Alignment":
// N = batch max_seqlen) and written in fp32.  The LayerNorm over the H*d_v features of a token
// and the U gating ("Similar shape, different aggregation": U_i (.) Norm(sum_j A_ij V_j)) run in
// ln_gate_kernel, one warp per token.
#include "kernels.h"

namespace hstu {

namespace {

constexpr int kThreads = 256;
constexpr int kFwdBM = 64, kFwdBN = 64;
constexpr int kBwdBM = 32, kBwdBN = 32;
constexpr int kMaxColsPerThread = 16;   // d <= 256 with 16 threads across a row
constexpr int kRelHistMax = 8192;       // rel-bias gradient histogram kept in shared memory

struct SmemHeader {
    uint64_t thr[kMaxTimeBuckets];
    float tb[kMaxTimeBuckets];
};

__device__ __forceinline__ void load_header(const DevParams &p, SmemHeader *hd)
{
    for (int x = threadIdx.x; x < p.n_thr; x += blockDim.x) hd->thr[x] = p.thr[x];
    for (int x = threadIdx.x; x < p.NB; x += blockDim.x) hd->tb[x] = p.tb[x];
}

// Bias of local positions i, j; also returns the table indices (-1 when absent).
__device__ __forceinline__ float pair_bias(const DevParams &p, const SmemHeader *hd,
                                           const SeqInfo &s, int pi, int pj, int64_t tsi,
                                           int64_t tsj, int *ri, int *bk)
{
    float b = 0.f;
    *ri = -1;
    *bk = -1;
    if (p.R > 0) {
        int r = pi - pj;
        r = rel_index(r, p.R, (p.flags & HSTU_FLAG_REL_ABS) != 0);
        *ri = r;
        b += __ldg(p.rel + r);
    }
    if (p.NB > 0) {
        int k = bucket_search(hd->thr, p.n_thr, abs_diff_u64(tsi, tsj));
        *bk = k;
        b += hd->tb[k];
    }
    return b;
}

template <typename T>
__device__ __forceinline__ void load_tile(float *dst, int ld, const T *src, int64_t row0,
                                          int rows_valid, int rows, int H, int h, int d)
{
    for (int x = threadIdx.x; x < rows * d; x += blockDim.x) {
        int r = x / d, e = x - r * d;
        float val = 0.f;
        if (r < rows_valid) val = to_f32<T>(src[((row0 + r) * H + h) * (int64_t)d + e]);
        dst[r * ld + e] = val;
    }
}

}  // namespace

size_t simt_fwd_smem_bytes(int dqk, int dv)
{
    return sizeof(SmemHeader) + sizeof(int64_t) * (kFwdBM + kFwdBN) +
           sizeof(float) * ((size_t)kFwdBM * (dqk + 1) + (size_t)kFwdBN * (dqk + 1) +
                            (size_t)kFwdBN * (dv + 1) + (size_t)kFwdBM * (kFwdBN + 1));
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    fwd_simt_kernel(const __grid_constant__ DevParams p, const T *__restrict__ q,
                    const T *__restrict__ k, const T *__restrict__ v, float *__restrict__ y)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SmemHeader *hd = reinterpret_cast<SmemHeader *>(smem_raw);
    int64_t *tsq = reinterpret_cast<int64_t *>(hd + 1);
    int64_t *tsk = tsq + kFwdBM;
    const int dqk = p.dqk, dv = p.dv, H = p.H;
    const int ldq = dqk + 1, ldv = dv + 1, ldp = kFwdBN + 1;
    float *Qs = reinterpret_cast<float *>(tsk + kFwdBN);
    float *Ks = Qs + kFwdBM * ldq;
    float *Vs = Ks + kFwdBN * ldq;
    float *Ps = Vs + kFwdBN * ldv;

    const int qt = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const SeqInfo s = load_seq(p, b, qt == 0 && h == 0 && threadIdx.x == 0);
    if (qt == 0 && h == 0) {   // rows no block writes: zero Y
        RowRange rr[3];
        const int n = skipped_rows(p, b, rr);
        for (int x = 0; x < n; ++x) zero_rows(y, p.D, rr[x], threadIdx.x, kThreads);
    }
    const int i0 = qt * kFwdBM;
    if (i0 >= s.L) return;
    if ((p.flags & HSTU_FLAG_CANDIDATES_ONLY) && i0 + kFwdBM <= s.E) return;   // no candidate row
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

    load_header(p, hd);
    const int qrows = min(kFwdBM, s.L - i0);
    load_tile<T>(Qs, ldq, q, s.start + i0, qrows, kFwdBM, H, h, dqk);
    if (p.NB > 0)
        for (int r = tid; r < kFwdBM; r += kThreads)
            tsq[r] = (i0 + r < s.L) ? p.ts[s.start + clamp_pos(i0 + r, s.E)] : 0;

    float acc[4][kMaxColsPerThread];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int n = 0; n < kMaxColsPerThread; ++n) acc[m][n] = 0.f;

    const int nkt = (s.L + kFwdBN - 1) / kFwdBN;
    for (int kt = 0; kt < nkt; ++kt) {
        const int j0 = kt * kFwdBN;
        if (!tile_any_valid(i0, i0 + kFwdBM - 1, j0, j0 + kFwdBN - 1, s, p.W)) continue;
        __syncthreads();   // previous tile's Ks/Vs/Ps fully consumed
        const int krows = min(kFwdBN, s.L - j0);
        load_tile<T>(Ks, ldq, k, s.start + j0, krows, kFwdBN, H, h, dqk);
        load_tile<T>(Vs, ldv, v, s.start + j0, krows, kFwdBN, H, h, dv);
        if (p.NB > 0)
            for (int c = tid; c < kFwdBN; c += kThreads)
                tsk[c] = (j0 + c < s.L) ? p.ts[s.start + clamp_pos(j0 + c, s.E)] : 0;
        __syncthreads();

        float sacc[4][4];
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) sacc[m][n] = 0.f;
        for (int e = 0; e < dqk; ++e) {
            float a[4], bb[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) a[m] = Qs[(ty + 16 * m) * ldq + e];
#pragma unroll
            for (int n = 0; n < 4; ++n) bb[n] = Ks[(tx + 16 * n) * ldq + e];
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int n = 0; n < 4; ++n) sacc[m][n] = fmaf(a[m], bb[n], sacc[m][n]);
        }
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int n = 0; n < 4; ++n) {
                const int r = ty + 16 * m, c = tx + 16 * n;
                const int i = i0 + r, j = j0 + c;
                float a = 0.f;
                if (i < s.L && j < s.L && pair_valid(i, j, s, p.W)) {
                    int ri, bk;
                    float bias = pair_bias(p, hd, s, clamp_pos(i, s.E), clamp_pos(j, s.E),
                                           p.NB > 0 ? tsq[r] : 0, p.NB > 0 ? tsk[c] : 0, &ri,
                                           &bk);
                    a = silu_f32(fmaf(p.alpha, sacc[m][n], bias));
                }
                Ps[r * ldp + c] = a;
            }
        __syncthreads();

        for (int jj = 0; jj < kFwdBN; ++jj) {
            float pv[4];
#pragma unroll
            for (int m = 0; m < 4; ++m) pv[m] = Ps[(ty + 16 * m) * ldp + jj];
#pragma unroll
            for (int n = 0; n < kMaxColsPerThread; ++n) {
                const int cc = tx + 16 * n;
                if (cc < dv) {
                    const float vv = Vs[jj * ldv + cc];
#pragma unroll
                    for (int m = 0; m < 4; ++m) acc[m][n] = fmaf(pv[m], vv, acc[m][n]);
                }
            }
        }
    }

    const int D = p.D;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const int i = i0 + ty + 16 * m;
        if (i >= s.L) continue;
        float *yr = y + (s.start + i) * (int64_t)D + h * dv;
#pragma unroll
        for (int n = 0; n < kMaxColsPerThread; ++n) {
            const int cc = tx + 16 * n;
            if (cc < dv) yr[cc] = acc[m][n] * p.inv_N;
        }
    }
}

// One warp per token: mean and biased variance over the D features (two passes in
// registers), Zhat = (Y - mean) * rstd, out = U (.) Zhat.
template <typename T>
__global__ void __launch_bounds__(kThreads)
    ln_gate_kernel(const __grid_constant__ DevParams p, const float *__restrict__ y,
                   const T *__restrict__ u, T *__restrict__ out, float *__restrict__ mean_out,
                   float *__restrict__ rstd_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    if (row >= p.T) return;
    const int D = p.D;
    const float *yr = y + row * D;
    float vals[64];
    float sum = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const int e = lane + 32 * c;
        vals[c] = e < D ? yr[e] : 0.f;
        sum += vals[c];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float mu = sum / (float)D;
    float sq = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const int e = lane + 32 * c;
        const float dlt = e < D ? vals[c] - mu : 0.f;
        sq = fmaf(dlt, dlt, sq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    const float rs = rsqrtf(sq / (float)D + p.eps);
    const T *ur = u + row * D;
    T *orow = out + row * D;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const int e = lane + 32 * c;
        if (e < D) orow[e] = from_f32<T>(to_f32<T>(ur[e]) * ((vals[c] - mu) * rs));
    }
    if (lane == 0 && mean_out) {
        mean_out[row] = mu;
        rstd_out[row] = rs;
    }
}

// One warp per token: dU = dO (.) Zhat, dZ = dO (.) U,
// dY = rstd * (dZ - mean(dZ) - Zhat * mean(dZ (.) Zhat)).
// With DYT = bf16, dY is written as a pair of bf16 arrays, hi = bf16(dY) at dy and
// lo = bf16(dY - hi) at dy + T*D, so that tensor-core products with dY keep about 16
// significant bits (LayerNorm makes dY orthogonal to Y, and sums over dY can cancel).
template <typename T, typename DYT>
__global__ void __launch_bounds__(kThreads)
    ln_gate_bwd_kernel(const __grid_constant__ DevParams p, const T *__restrict__ dout,
                       const T *__restrict__ u, const float *__restrict__ y,
                       const float *__restrict__ mean, const float *__restrict__ rstd,
                       T *__restrict__ du, DYT *__restrict__ dy, const BwdZero zj)
{
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5);
    bwd_zero_small(zj);
    if (row >= p.T) return;
    bwd_zero_row(zj, row, lane);
    const int D = p.D;
    const float mu = mean[row], rs = rstd[row];
    float z[64], dz[64];
    float m1 = 0.f, m2 = 0.f;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const int e = lane + 32 * c;
        z[c] = 0.f;
        dz[c] = 0.f;
        if (e < D) {
            const float zz = (y[row * D + e] - mu) * rs;
            const float g = to_f32<T>(dout[row * D + e]);
            z[c] = zz;
            dz[c] = g * to_f32<T>(u[row * D + e]);
            du[row * D + e] = from_f32<T>(g * zz);
        }
        m1 += dz[c];
        m2 = fmaf(dz[c], z[c], m2);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        m1 += __shfl_xor_sync(0xffffffffu, m1, o);
        m2 += __shfl_xor_sync(0xffffffffu, m2, o);
    }
    m1 /= (float)D;
    m2 /= (float)D;
#pragma unroll
    for (int c = 0; c < 64; ++c) {
        const int e = lane + 32 * c;
        if (e < D) {
            const float g = rs * (dz[c] - m1 - z[c] * m2);
            const DYT hi = from_f32<DYT>(g);
            dy[row * D + e] = hi;
            if (sizeof(DYT) == 2) dy[p.T * D + row * D + e] = from_f32<DYT>(g - to_f32<DYT>(hi));
        }
    }
}

size_t simt_bwd_smem_bytes(int dqk, int dv, int R)
{
    size_t n = sizeof(SmemHeader) + sizeof(int64_t) * (kBwdBM + kBwdBN);
    n += sizeof(float) * ((size_t)kBwdBN * (dqk + 1) + (size_t)kBwdBN * (dv + 1) +
                          (size_t)kBwdBM * (dqk + 1) + (size_t)kBwdBM * (dv + 1) +
                          3 * (size_t)kBwdBM * (kBwdBN + 1));
    n += sizeof(float) * (size_t)(R <= kRelHistMax ? R : 0) + sizeof(float) * kMaxTimeBuckets;
    return n;
}

// Backward per (sequence, head, 32-key tile): over every 32-row query tile that sees the
// keys, recompute S and A, then
//   dV_j += sum_i A_ij dY_i;  dA_ij = <dY_i, V_j>;  dS_ij = mask * dA_ij * SiLU'(s_ij) / N;
//   dK_j += alpha sum_i dS_ij Q_i;  dQ_i += alpha sum_j dS_ij K_j (fp32 atomics);
//   d rel[r_ij] += dS_ij;  d tb[bucket_ij] += dS_ij (shared-memory histograms, then atomics).
template <typename T>
__global__ void __launch_bounds__(kThreads)
    bwd_simt_kernel(const __grid_constant__ DevParams p, const T *__restrict__ q,
                    const T *__restrict__ k, const T *__restrict__ v,
                    const float *__restrict__ dy, float *__restrict__ dq_acc, T *__restrict__ dk,
                    T *__restrict__ dv_out, float *__restrict__ d_rel, float *__restrict__ d_tb)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SmemHeader *hd = reinterpret_cast<SmemHeader *>(smem_raw);
    int64_t *tsq = reinterpret_cast<int64_t *>(hd + 1);
    int64_t *tsk = tsq + kBwdBM;
    const int dqk = p.dqk, dv = p.dv, H = p.H, D = p.D;
    const int ldq = dqk + 1, ldv = dv + 1, lds = kBwdBN + 1;
    float *Ks = reinterpret_cast<float *>(tsk + kBwdBN);
    float *Vs = Ks + kBwdBN * ldq;
    float *Qs = Vs + kBwdBN * ldv;
    float *dYs = Qs + kBwdBM * ldq;
    float *As = dYs + kBwdBM * ldv;
    float *Gs = As + kBwdBM * lds;
    float *DSs = Gs + kBwdBM * lds;
    const bool rel_in_smem = p.R <= kRelHistMax;
    float *hrel = DSs + kBwdBM * lds;
    float *htb = hrel + (rel_in_smem ? p.R : 0);

    const int kt = blockIdx.x, b = blockIdx.y, h = blockIdx.z;
    const SeqInfo s = load_seq(p, b, kt == 0 && h == 0 && threadIdx.x == 0);
    if (kt == 0 && h == 0) {   // rows no block writes: zero dK, dV
        RowRange rr[3];
        const int n = skipped_rows(p, b, rr);
        for (int x = 0; x < n; ++x) {
            zero_rows(dk, (int64_t)H * dqk, rr[x], threadIdx.x, kThreads);
            zero_rows(dv_out, (int64_t)H * dv, rr[x], threadIdx.x, kThreads);
        }
    }
    const int j0 = kt * kBwdBN;
    if (j0 >= s.L) return;
    const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;

    load_header(p, hd);
    if (rel_in_smem)
        for (int x = tid; x < p.R; x += kThreads) hrel[x] = 0.f;
    for (int x = tid; x < p.NB; x += kThreads) htb[x] = 0.f;
    const int krows = min(kBwdBN, s.L - j0);
    load_tile<T>(Ks, ldq, k, s.start + j0, krows, kBwdBN, H, h, dqk);
    load_tile<T>(Vs, ldv, v, s.start + j0, krows, kBwdBN, H, h, dv);
    if (p.NB > 0)
        for (int c = tid; c < kBwdBN; c += kThreads)
            tsk[c] = (j0 + c < s.L) ? p.ts[s.start + clamp_pos(j0 + c, s.E)] : 0;

    float dk_acc[2][kMaxColsPerThread], dv_acc[2][kMaxColsPerThread];
#pragma unroll
    for (int m = 0; m < 2; ++m)
#pragma unroll
        for (int n = 0; n < kMaxColsPerThread; ++n) dk_acc[m][n] = dv_acc[m][n] = 0.f;

    const int nqt = (s.L + kBwdBM - 1) / kBwdBM;
    for (int qt = 0; qt < nqt; ++qt) {
        const int i0 = qt * kBwdBM;
        if (!tile_any_valid(i0, i0 + kBwdBM - 1, j0, j0 + kBwdBN - 1, s, p.W)) continue;
        __syncthreads();
        const int qrows = min(kBwdBM, s.L - i0);
        load_tile<T>(Qs, ldq, q, s.start + i0, qrows, kBwdBM, H, h, dqk);
        for (int x = tid; x < kBwdBM * dv; x += kThreads) {
            int r = x / dv, e = x - r * dv;
            dYs[r * ldv + e] = r < qrows ? dy[(s.start + i0 + r) * (int64_t)D + h * dv + e] : 0.f;
        }
        if (p.NB > 0)
            for (int r = tid; r < kBwdBM; r += kThreads)
                tsq[r] = (i0 + r < s.L) ? p.ts[s.start + clamp_pos(i0 + r, s.E)] : 0;
        __syncthreads();

        // S = Q K^T and dA = dY V^T for this thread's 2x2 pairs
        float sacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}}, dacc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
        for (int e = 0; e < dqk; ++e) {
            const float a0 = Qs[ty * ldq + e], a1 = Qs[(ty + 16) * ldq + e];
            const float b0 = Ks[tx * ldq + e], b1 = Ks[(tx + 16) * ldq + e];
            sacc[0][0] = fmaf(a0, b0, sacc[0][0]);
            sacc[0][1] = fmaf(a0, b1, sacc[0][1]);
            sacc[1][0] = fmaf(a1, b0, sacc[1][0]);
            sacc[1][1] = fmaf(a1, b1, sacc[1][1]);
        }
        for (int e = 0; e < dv; ++e) {
            const float a0 = dYs[ty * ldv + e], a1 = dYs[(ty + 16) * ldv + e];
            const float b0 = Vs[tx * ldv + e], b1 = Vs[(tx + 16) * ldv + e];
            dacc[0][0] = fmaf(a0, b0, dacc[0][0]);
            dacc[0][1] = fmaf(a0, b1, dacc[0][1]);
            dacc[1][0] = fmaf(a1, b0, dacc[1][0]);
            dacc[1][1] = fmaf(a1, b1, dacc[1][1]);
        }
#pragma unroll
        for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int n = 0; n < 2; ++n) {
                const int r = ty + 16 * m, c = tx + 16 * n;
                const int i = i0 + r, j = j0 + c;
                float a = 0.f, ds = 0.f;
                if (i < s.L && j < s.L && pair_valid(i, j, s, p.W)) {
                    int ri, bk;
                    const float bias =
                        pair_bias(p, hd, s, clamp_pos(i, s.E), clamp_pos(j, s.E),
                                  p.NB > 0 ? tsq[r] : 0, p.NB > 0 ? tsk[c] : 0, &ri, &bk);
                    const float sv = fmaf(p.alpha, sacc[m][n], bias);
                    a = silu_f32(sv) * p.inv_N;
                    ds = dacc[m][n] * silu_grad_f32(sv) * p.inv_N;
                    if (ri >= 0) {
                        if (rel_in_smem) atomicAdd(hrel + ri, ds);
                        else atomicAdd(d_rel + ri, ds);
                    }
                    if (bk >= 0) atomicAdd(htb + bk, ds);
                }
                As[r * lds + c] = a;
                DSs[r * lds + c] = ds;
            }
        __syncthreads();

        // dV_j += sum_i A_ij dY_i ; dK_j += alpha sum_i dS_ij Q_i   (rows j = ty, ty+16)
        for (int r = 0; r < kBwdBM; ++r) {
            const float a0 = As[r * lds + ty], a1 = As[r * lds + ty + 16];
            const float s0 = DSs[r * lds + ty], s1 = DSs[r * lds + ty + 16];
#pragma unroll
            for (int n = 0; n < kMaxColsPerThread; ++n) {
                const int cc = tx + 16 * n;
                if (cc < dv) {
                    const float g = dYs[r * ldv + cc];
                    dv_acc[0][n] = fmaf(a0, g, dv_acc[0][n]);
                    dv_acc[1][n] = fmaf(a1, g, dv_acc[1][n]);
                }
                if (cc < dqk) {
                    const float qq = Qs[r * ldq + cc];
                    dk_acc[0][n] = fmaf(s0, qq, dk_acc[0][n]);
                    dk_acc[1][n] = fmaf(s1, qq, dk_acc[1][n]);
                }
            }
        }
        // dQ_i += alpha sum_j dS_ij K_j   (rows i = ty, ty+16)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int r = ty + 16 * m;
            if (r >= qrows) continue;
            float *dqr = dq_acc + ((s.start + i0 + r) * H + h) * (int64_t)dqk;
#pragma unroll
            for (int n = 0; n < kMaxColsPerThread; ++n) {
                const int cc = tx + 16 * n;
                if (cc < dqk) {
                    float accq = 0.f;
                    for (int c = 0; c < kBwdBN; ++c)
                        accq = fmaf(DSs[r * lds + c], Ks[c * ldq + cc], accq);
                    if (accq != 0.f) atomicAdd(dqr + cc, p.alpha * accq);
                }
            }
        }
    }

#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int c = ty + 16 * m;
        if (c >= krows) continue;
        T *dkr = dk + ((s.start + j0 + c) * H + h) * (int64_t)dqk;
        T *dvr = dv_out + ((s.start + j0 + c) * H + h) * (int64_t)dv;
#pragma unroll
        for (int n = 0; n < kMaxColsPerThread; ++n) {
            const int cc = tx + 16 * n;
            if (cc < dqk) dkr[cc] = from_f32<T>(p.alpha * dk_acc[m][n]);
            if (cc < dv) dvr[cc] = from_f32<T>(dv_acc[m][n]);
        }
    }
    __syncthreads();
    if (rel_in_smem)
        for (int x = tid; x < p.R; x += kThreads)
            if (hrel[x] != 0.f) atomicAdd(d_rel + x, hrel[x]);
    for (int x = tid; x < p.NB; x += kThreads)
        if (htb[x] != 0.f) atomicAdd(d_tb + x, htb[x]);
}

template <typename T>
__global__ void convert_kernel(const float *__restrict__ src, T *__restrict__ dst, int64_t n)
{
    grid_dep_wait();   // src is complete once the kernel ahead on the stream is
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n;
         x += (int64_t)gridDim.x * blockDim.x)
        dst[x] = from_f32<T>(src[x]);
}

// ------------------------------------------------------------------ launchers

template <typename T>
cudaError_t launch_simt_fwd(const DevParams &p, const void *q, const void *k, const void *v,
                            float *y, cudaStream_t st)
{
    const size_t smem = simt_fwd_smem_bytes(p.dqk, p.dv);
    cudaError_t e = cudaFuncSetAttribute(fwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.N + kFwdBM - 1) / kFwdBM, p.B, p.H);
    fwd_simt_kernel<T><<<grid, kThreads, smem, st>>>(p, (const T *)q, (const T *)k,
                                                     (const T *)v, y);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ln_gate(const DevParams &p, const float *y, const void *u, void *out,
                           float *mean, float *rstd, cudaStream_t st)
{
    if (ln_vec_supported(p.D)) return launch_ln_gate_vec<T>(p, y, u, out, mean, rstd, st);
    const int rows_per_block = kThreads / 32;
    const int64_t blocks = (p.T + rows_per_block - 1) / rows_per_block;
    ln_gate_kernel<T><<<(unsigned)blocks, kThreads, 0, st>>>(p, y, (const T *)u, (T *)out, mean,
                                                             rstd);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_ln_gate_bwd(const DevParams &p, const void *dout, const void *u,
                               const float *y, const float *mean, const float *rstd, void *du,
                               void *dy, bool dy_bf16, const BwdZero &zero, cudaStream_t st)
{
    if (ln_vec_supported(p.D))
        return launch_ln_gate_bwd_vec<T>(p, dout, u, y, mean, rstd, du, dy, dy_bf16, zero, st);
    const int rows_per_block = kThreads / 32;
    const int64_t blocks = (p.T + rows_per_block - 1) / rows_per_block;
    if (dy_bf16)
        ln_gate_bwd_kernel<T, __nv_bfloat16><<<(unsigned)blocks, kThreads, 0, st>>>(
            p, (const T *)dout, (const T *)u, y, mean, rstd, (T *)du, (__nv_bfloat16 *)dy, zero);
    else
        ln_gate_bwd_kernel<T, float><<<(unsigned)blocks, kThreads, 0, st>>>(
            p, (const T *)dout, (const T *)u, y, mean, rstd, (T *)du, (float *)dy, zero);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_simt_bwd(const DevParams &p, const void *q, const void *k, const void *v,
                            const float *dy, float *dq_acc, void *dk, void *dv, float *d_rel,
                            float *d_tb, cudaStream_t st)
{
    const size_t smem = simt_bwd_smem_bytes(p.dqk, p.dv, p.R);
    cudaError_t e = cudaFuncSetAttribute(bwd_simt_kernel<T>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((p.N + kBwdBN - 1) / kBwdBN, p.B, p.H);
    bwd_simt_kernel<T><<<grid, kThreads, smem, st>>>(p, (const T *)q, (const T *)k, (const T *)v,
                                                     dy, dq_acc, (T *)dk, (T *)dv, d_rel, d_tb);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_convert(const float *src, void *dst, int64_t n, cudaStream_t st)
{
    if (n <= 0) return cudaSuccess;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    return launch_pdl(convert_kernel<T>, dim3((unsigned)blocks), dim3(256), 0, st, src, (T *)dst,
                      n);
}

template cudaError_t launch_simt_fwd<float>(const DevParams &, const void *, const void *,
                                            const void *, float *, cudaStream_t);
template cudaError_t launch_simt_fwd<__nv_bfloat16>(const DevParams &, const void *,
                                                    const void *, const void *, float *,
                                                    cudaStream_t);
template cudaError_t launch_ln_gate<float>(const DevParams &, const float *, const void *,
                                           void *, float *, float *, cudaStream_t);
template cudaError_t launch_ln_gate<__nv_bfloat16>(const DevParams &, const float *,
                                                   const void *, void *, float *, float *,
                                                   cudaStream_t);
template cudaError_t launch_ln_gate_bwd<float>(const DevParams &, const void *, const void *,
                                               const float *, const float *, const float *,
                                               void *, void *, bool, const BwdZero &,
                                               cudaStream_t);
template cudaError_t launch_ln_gate_bwd<__nv_bfloat16>(const DevParams &, const void *,
                                                       const void *, const float *,
                                                       const float *, const float *, void *,
                                                       void *, bool, const BwdZero &,
                                                       cudaStream_t);
template cudaError_t launch_simt_bwd<float>(const DevParams &, const void *, const void *,
                                            const void *, const float *, float *, void *, void *,
                                            float *, float *, cudaStream_t);
template cudaError_t launch_simt_bwd<__nv_bfloat16>(const DevParams &, const void *,
                                                    const void *, const void *, const float *,
                                                    float *, void *, void *, float *, float *,
                                                    cudaStream_t);
template cudaError_t launch_convert<__nv_bfloat16>(const float *, void *, int64_t,
                                                   cudaStream_t);

}  // namespace hstu
