// wkv6_backward.cu -- Eagle/Finch WKV-6 backward pass (gradients for training), fp32 on
// CUDA cores.
//
// Source: "RWKV-5/6 (Eagle and Finch)", section 4.1.2 (time mixing: S is a sum of k^T v,
// each key channel decayed by w every step, gain u on the current token, receptance r
// applied like a query; w = exp(-exp(omega))) and section 4.2.2 (Finch: w_t per token).
// Forward, per (b, h) and token t, with S the state before t:
//   o_t[j] = sum_i r_t[i] (S[i][j] + u[i] k_t[i] v_t[j]),   S <- diag(w_t) S + k_t^T v_t.
// With L = dL/dS for the state after t (dsT after the last token), the chain rule gives
//   dr_t[i] = sum_j do_t[j] S[i][j] + u[i] k_t[i] (do_t . v_t)
//   dk_t[i] = sum_j L[i][j] v_t[j] + u[i] r_t[i] (do_t . v_t)
//   dv_t[j] = sum_i L[i][j] k_t[i] + (sum_i r_t[i] u[i] k_t[i]) do_t[j]
//   dw_t[i] = sum_j L[i][j] S[i][j]
//   du[i]  += r_t[i] k_t[i] (do_t . v_t)
//   L <- diag(w_t) L + r_t^T do_t         (the gradient of the state before t)
// and ds0 = L once token 0 is undone.  With the decay given by its logit,
// domega_t = dw_t * (-exp(omega_t) w_t).
//
// Each term is a dot product along one axis of a 64 x 64 matrix, so each kernel keeps the
// matrix it walks in registers with that axis local to a thread pair:
//   wkv6_bwd_forward_kernel  rows of S (thread pair per key channel i), forward in time:
//                            dr, du, and a checkpoint of S every kBlock tokens;
//   wkv6_bwd_rows_kernel     rows of L, backward in time: dk and dw.  dw needs the state
//                            before every token: each block of kBlock tokens is recomputed
//                            forward from its checkpoint into shared memory first;
//   wkv6_bwd_cols_kernel     columns of L (thread pair per value channel j), backward in
//                            time: dv and ds0;
//   wkv6_bwd_du_kernel       du summed over the batch rows (fixed order: deterministic).
// One CTA of 128 threads per (b, h).  A thread pair shares one row (or column) and splits
// its 64 entries into interleaved float4 groups (pair half p owns entries 8m + 4p .. +3), so
// the pair's shared-memory reads of a broadcast vector fall in different banks.
#include "wkv_internal.cuh"

#include <algorithm>

namespace wkv {
namespace {

constexpr int kN = 64;
constexpr int kThreads = 128;
constexpr int kBlock = 8;  // tokens per checkpoint
constexpr int kStashBytes = kBlock * kThreads * 32 * 4;  // states of one block, per CTA

template <typename T> __device__ __forceinline__ float ldf(const T *p);
template <> __device__ __forceinline__ float ldf<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}

// Decay from its logit, w = exp(-exp(omega)), with the accurate exponential.
__device__ __forceinline__ float decay(float x, bool omega) { return omega ? expf(-expf(x)) : x; }

__device__ __forceinline__ float pair_sum(float x) { return x + __shfl_xor_sync(0xffffffffu, x, 1); }

// index of the e-th entry of group m owned by pair half p
__device__ __forceinline__ int col(int m, int p, int e) { return 8 * m + 4 * p + e; }

// ------------------------------------------------------------------ forward: dr, du, checkpoints
template <typename T>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_forward_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                        const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                        const float *__restrict__ s0, const T *__restrict__ dy, float *__restrict__ dr,
                        float *__restrict__ ckpt, float *__restrict__ du_part, int omega)
{
    __shared__ __align__(16) float vs[2][kN], gs[2][kN];
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    const int tid = threadIdx.x, i = tid >> 1, p = tid & 1;
    const int64_t nblk = (Tlen + kBlock - 1) / kBlock;
    const float ui = u[h * kN + i];

    float S[32];
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) S[4 * m + e] = s0 ? s0[n * kN * kN + i * kN + col(m, p, e)] : 0.f;

    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;
    float du_acc = 0.f;
    for (int64_t t = 0; t < Tlen; ++t) {
        const int buf = static_cast<int>(t & 1);
        const int64_t o = base + t * stride;
        if (tid < kN) vs[buf][tid] = ldf(v + o + tid);
        else gs[buf][tid - kN] = ldf(dy + o + tid - kN);
        const float ri = ldf(r + o + i), ki = ldf(k + o + i), wi = decay(ldf(w + o + i), omega);
        if (t % kBlock == 0) {  // checkpoint: the state before this token, in register order
            float4 *cp = reinterpret_cast<float4 *>(ckpt + (n * nblk + t / kBlock) * (kN * kN));
#pragma unroll
            for (int m = 0; m < 8; ++m)
                cp[m * kThreads + tid] = make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
        }
        __syncthreads();
        float sd = 0.f, dot = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 g4 = *reinterpret_cast<const float4 *>(&gs[buf][col(m, p, 0)]);
            const float4 v4 = *reinterpret_cast<const float4 *>(&vs[buf][col(m, p, 0)]);
            sd = fmaf(S[4 * m], g4.x, sd);
            sd = fmaf(S[4 * m + 1], g4.y, sd);
            sd = fmaf(S[4 * m + 2], g4.z, sd);
            sd = fmaf(S[4 * m + 3], g4.w, sd);
            dot = fmaf(g4.x, v4.x, dot);
            dot = fmaf(g4.y, v4.y, dot);
            dot = fmaf(g4.z, v4.z, dot);
            dot = fmaf(g4.w, v4.w, dot);
            S[4 * m] = fmaf(wi, S[4 * m], ki * v4.x);
            S[4 * m + 1] = fmaf(wi, S[4 * m + 1], ki * v4.y);
            S[4 * m + 2] = fmaf(wi, S[4 * m + 2], ki * v4.z);
            S[4 * m + 3] = fmaf(wi, S[4 * m + 3], ki * v4.w);
        }
        sd = pair_sum(sd);
        dot = pair_sum(dot);
        if (p == 0) dr[o + i] = fmaf(ui * ki, dot, sd);
        du_acc = fmaf(ri * ki, dot, du_acc);
    }
    if (p == 0) du_part[n * kN + i] = du_acc;
}

// ------------------------------------------------------------------ backward, rows: dk, dw
template <typename T>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_rows_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                     const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                     const T *__restrict__ dy, const float *__restrict__ dsT, const float *__restrict__ ckpt,
                     float *__restrict__ dk, float *__restrict__ dw, int omega)
{
    extern __shared__ __align__(16) unsigned char smem[];
    float4 *stash = reinterpret_cast<float4 *>(smem);                                // [kBlock][8][kThreads]
    float *vs = reinterpret_cast<float *>(smem + kStashBytes);                       // [kBlock][kN]
    float *gs = vs + kBlock * kN;                                                    // [kBlock][kN]
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    const int tid = threadIdx.x, i = tid >> 1, p = tid & 1;
    const int64_t nblk = (Tlen + kBlock - 1) / kBlock;
    const float ui = u[h * kN + i];
    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;

    float L[32];
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) L[4 * m + e] = dsT ? dsT[n * kN * kN + i * kN + col(m, p, e)] : 0.f;

    for (int64_t c = nblk - 1; c >= 0; --c) {
        const int64_t t0 = c * kBlock;
        const int tv = static_cast<int>(std::min<int64_t>(kBlock, Tlen - t0));
        __syncthreads();  // the previous block's v, do are no longer read
        for (int q = tid; q < 2 * kBlock * kN; q += kThreads) {
            const int tt = q / (2 * kN), x = q % (2 * kN);
            float val = 0.f;
            if (tt < tv) {
                const int64_t o = base + (t0 + tt) * stride;
                val = x < kN ? ldf(v + o + x) : ldf(dy + o + x - kN);
            }
            (x < kN ? vs : gs)[tt * kN + (x % kN)] = val;
        }
        float rr[kBlock], kk[kBlock], ww[kBlock], om[kBlock];
#pragma unroll
        for (int m = 0; m < kBlock; ++m) {
            rr[m] = kk[m] = om[m] = 0.f;
            ww[m] = 1.f;
            if (m < tv) {
                const int64_t o = base + (t0 + m) * stride + i;
                rr[m] = ldf(r + o);
                kk[m] = ldf(k + o);
                om[m] = ldf(w + o);
                ww[m] = decay(om[m], omega);
            }
        }
        // the states before each token of the block, from the checkpoint (own entries only)
        const float4 *cp = reinterpret_cast<const float4 *>(ckpt + (n * nblk + c) * (kN * kN));
        float s[32];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 x = cp[m * kThreads + tid];
            s[4 * m] = x.x;
            s[4 * m + 1] = x.y;
            s[4 * m + 2] = x.z;
            s[4 * m + 3] = x.w;
        }
        __syncthreads();  // v, do of the block in shared memory
#pragma unroll
        for (int tt = 0; tt < kBlock; ++tt) {
            if (tt < tv) {
#pragma unroll
                for (int m = 0; m < 8; ++m)
                    stash[(tt * 8 + m) * kThreads + tid] =
                        make_float4(s[4 * m], s[4 * m + 1], s[4 * m + 2], s[4 * m + 3]);
                if (tt + 1 < tv) {
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        const float4 v4 = *reinterpret_cast<const float4 *>(&vs[tt * kN + col(m, p, 0)]);
                        s[4 * m] = fmaf(ww[tt], s[4 * m], kk[tt] * v4.x);
                        s[4 * m + 1] = fmaf(ww[tt], s[4 * m + 1], kk[tt] * v4.y);
                        s[4 * m + 2] = fmaf(ww[tt], s[4 * m + 2], kk[tt] * v4.z);
                        s[4 * m + 3] = fmaf(ww[tt], s[4 * m + 3], kk[tt] * v4.w);
                    }
                }
            }
        }
#pragma unroll
        for (int tt = kBlock - 1; tt >= 0; --tt) {
            if (tt < tv) {
                float dwp = 0.f, dkp = 0.f, dot = 0.f;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const float4 s4 = stash[(tt * 8 + m) * kThreads + tid];
                    const float4 v4 = *reinterpret_cast<const float4 *>(&vs[tt * kN + col(m, p, 0)]);
                    const float4 g4 = *reinterpret_cast<const float4 *>(&gs[tt * kN + col(m, p, 0)]);
                    dwp = fmaf(L[4 * m], s4.x, dwp);
                    dwp = fmaf(L[4 * m + 1], s4.y, dwp);
                    dwp = fmaf(L[4 * m + 2], s4.z, dwp);
                    dwp = fmaf(L[4 * m + 3], s4.w, dwp);
                    dkp = fmaf(L[4 * m], v4.x, dkp);
                    dkp = fmaf(L[4 * m + 1], v4.y, dkp);
                    dkp = fmaf(L[4 * m + 2], v4.z, dkp);
                    dkp = fmaf(L[4 * m + 3], v4.w, dkp);
                    dot = fmaf(g4.x, v4.x, dot);
                    dot = fmaf(g4.y, v4.y, dot);
                    dot = fmaf(g4.z, v4.z, dot);
                    dot = fmaf(g4.w, v4.w, dot);
                    L[4 * m] = fmaf(ww[tt], L[4 * m], rr[tt] * g4.x);
                    L[4 * m + 1] = fmaf(ww[tt], L[4 * m + 1], rr[tt] * g4.y);
                    L[4 * m + 2] = fmaf(ww[tt], L[4 * m + 2], rr[tt] * g4.z);
                    L[4 * m + 3] = fmaf(ww[tt], L[4 * m + 3], rr[tt] * g4.w);
                }
                dwp = pair_sum(dwp);
                dkp = pair_sum(dkp);
                dot = pair_sum(dot);
                if (p == 0) {
                    const int64_t o = base + (t0 + tt) * stride + i;
                    dk[o] = fmaf(ui * rr[tt], dot, dkp);
                    // with the logit: dw/domega = -exp(omega) w
                    dw[o] = omega ? dwp * (-expf(om[tt]) * ww[tt]) : dwp;
                }
            }
        }
    }
}

// ------------------------------------------------------------------ backward, columns: dv, ds0
template <typename T>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_cols_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                     const T *__restrict__ w, const float *__restrict__ u, const T *__restrict__ dy,
                     const float *__restrict__ dsT, float *__restrict__ dv, float *__restrict__ ds0, int omega)
{
    __shared__ __align__(16) float rs[2][kN], ks[2][kN], ws[2][kN], rus[2][kN];
    __shared__ __align__(16) float us[kN];
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    const int tid = threadIdx.x, j = tid >> 1, p = tid & 1;
    if (tid < kN) us[tid] = u[h * kN + tid];
    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;

    // L[i][j] for this thread's rows i = col(m, p, e)
    float L[32];
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
        for (int e = 0; e < 4; ++e) L[4 * m + e] = dsT ? dsT[n * kN * kN + col(m, p, e) * kN + j] : 0.f;
    __syncthreads();

    for (int64_t t = Tlen - 1; t >= 0; --t) {
        const int buf = static_cast<int>(t & 1);
        const int64_t o = base + t * stride;
        if (tid < kN) {
            const float rv = ldf(r + o + tid);
            rs[buf][tid] = rv;
            rus[buf][tid] = rv * us[tid];
            ws[buf][tid] = decay(ldf(w + o + tid), omega);
        } else {
            ks[buf][tid - kN] = ldf(k + o + tid - kN);
        }
        const float gj = ldf(dy + o + j);
        __syncthreads();
        float dvp = 0.f, bon = 0.f;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const float4 k4 = *reinterpret_cast<const float4 *>(&ks[buf][col(m, p, 0)]);
            const float4 r4 = *reinterpret_cast<const float4 *>(&rs[buf][col(m, p, 0)]);
            const float4 w4 = *reinterpret_cast<const float4 *>(&ws[buf][col(m, p, 0)]);
            const float4 q4 = *reinterpret_cast<const float4 *>(&rus[buf][col(m, p, 0)]);
            dvp = fmaf(L[4 * m], k4.x, dvp);
            dvp = fmaf(L[4 * m + 1], k4.y, dvp);
            dvp = fmaf(L[4 * m + 2], k4.z, dvp);
            dvp = fmaf(L[4 * m + 3], k4.w, dvp);
            bon = fmaf(q4.x, k4.x, bon);
            bon = fmaf(q4.y, k4.y, bon);
            bon = fmaf(q4.z, k4.z, bon);
            bon = fmaf(q4.w, k4.w, bon);
            L[4 * m] = fmaf(w4.x, L[4 * m], r4.x * gj);
            L[4 * m + 1] = fmaf(w4.y, L[4 * m + 1], r4.y * gj);
            L[4 * m + 2] = fmaf(w4.z, L[4 * m + 2], r4.z * gj);
            L[4 * m + 3] = fmaf(w4.w, L[4 * m + 3], r4.w * gj);
        }
        dvp = pair_sum(dvp);
        bon = pair_sum(bon);
        if (p == 0) dv[o + j] = fmaf(bon, gj, dvp);
    }
    if (ds0) {
#pragma unroll
        for (int m = 0; m < 8; ++m)
#pragma unroll
            for (int e = 0; e < 4; ++e) ds0[n * kN * kN + col(m, p, e) * kN + j] = L[4 * m + e];
    }
}

// du[h][i] = sum over batch rows b of du_part[b][h][i], in order of b
__global__ void __launch_bounds__(kN) wkv6_bwd_du_kernel(int64_t B, int64_t H, const float *__restrict__ du_part,
                                                        float *__restrict__ du)
{
    const int64_t h = blockIdx.x;
    const int i = threadIdx.x;
    float acc = 0.f;
    for (int64_t b = 0; b < B; ++b) acc += du_part[(b * H + h) * kN + i];
    du[h * kN + i] = acc;
}

cudaError_t configure_rows()
{
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (done[dev]) return cudaSuccess;
    const int bytes = kStashBytes + 2 * kBlock * kN * 4;
    e = cudaFuncSetAttribute(wkv6_bwd_rows_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(wkv6_bwd_rows_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
    return cudaSuccess;
}

template <typename T>
cudaError_t launch_all(const Wkv6BwdArgs &a, cudaStream_t s)
{
    const int64_t bh = a.B * a.H;
    const int64_t nblk = (a.T + kBlock - 1) / kBlock;
    float *ckpt = static_cast<float *>(a.workspace);
    float *du_part = ckpt + bh * nblk * kN * kN;
    const int om = a.omega ? 1 : 0;
    const unsigned grid = static_cast<unsigned>(bh);
    const T *r = static_cast<const T *>(a.r), *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v), *w = static_cast<const T *>(a.w);
    const T *dy = static_cast<const T *>(a.dy);
    wkv6_bwd_forward_kernel<T><<<grid, kThreads, 0, s>>>(a.T, a.H, r, k, v, w, a.u, a.s0, dy, a.dr, ckpt,
                                                         du_part, om);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv6_bwd_rows_kernel<T><<<grid, kThreads, kStashBytes + 2 * kBlock * kN * 4, s>>>(
        a.T, a.H, r, k, v, w, a.u, dy, a.dsT, ckpt, a.dk, a.dw, om);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv6_bwd_cols_kernel<T><<<grid, kThreads, 0, s>>>(a.T, a.H, r, k, w, a.u, dy, a.dsT, a.dv, a.ds0, om);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv6_bwd_du_kernel<<<static_cast<unsigned>(a.H), kN, 0, s>>>(a.B, a.H, du_part, a.du);
    return cudaGetLastError();
}

}  // namespace

size_t wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H)
{
    const int64_t nblk = (T + kBlock - 1) / kBlock;
    return static_cast<size_t>(B * H) * static_cast<size_t>(nblk * kN * kN + kN) * sizeof(float);
}

cudaError_t wkv6_backward_launch(const Wkv6BwdArgs &a, cudaStream_t s)
{
    if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    if (a.B * a.H > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    cudaError_t e = configure_rows();
    if (e != cudaSuccess) return e;
    return a.bf16 ? launch_all<__nv_bfloat16>(a, s) : launch_all<float>(a, s);
}

}  // namespace wkv
