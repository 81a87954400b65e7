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
// matrix it walks in registers with that axis local to a group of TPR consecutive lanes:
//   wkv6_bwd_forward_kernel  rows of S, forward in time: dr, du, and a checkpoint of S
//                            every kBlock tokens;
//   wkv6_bwd_rows_kernel     rows of L, backward in time: dk and dw.  dw needs the state
//                            before every token: each block of kBlock tokens is recomputed
//                            forward from its checkpoint into shared memory first;
//   wkv6_bwd_cols_kernel     columns of L, backward in time: dv and ds0;
//   wkv6_bwd_du_kernel       du summed over the batch rows (fixed order: deterministic).
// Rows of S and of L evolve independently of one another (row i sees only w[i], k[i] or
// r[i]), and so do the columns of L, so each (b, h) is split over several CTAs of 128
// threads (TPR threads per row or column, 64 / TPR entries per thread).  Inputs reach
// shared memory 32 tokens at a time by cp.async, a chunk ahead of their use.
#include "wkv_internal.cuh"

#include <algorithm>
#include <mutex>

namespace wkv {
namespace {

constexpr int kN = 64;
constexpr int kThreads = 128;
constexpr int kBlock = 8;                 // tokens per checkpoint

// Decay from its logit, w = exp(-exp(omega)), with the accurate exponential.
__device__ __forceinline__ float decay(float x, bool omega) { return omega ? expf(-expf(x)) : x; }

// sum over the TPR consecutive lanes that share a row (or column)
template <int TPR> __device__ __forceinline__ float group_sum(float x)
{
#pragma unroll
    for (int m = 1; m < TPR; m <<= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// With TPR threads per row (or column), a thread owns E = 64 / TPR of its entries in float4
// groups: group m holds entries 4 TPR m + 4p .. + 3 for part p = lane % TPR.  The TPR parts
// of a row read a broadcast vector from disjoint bank groups.
template <int TPR> __device__ __forceinline__ int ent(int p, int e) { return 4 * TPR * (e >> 2) + 4 * p + (e & 3); }

// ------------------------------------------------------------------ staging in shared memory
// Inputs reach the kernels through shared memory, kChunk tokens at a time, copied with
// cp.async a whole chunk before their data is needed: the row walks alternate two copy
// buffers; the column walk widens each copied chunk into an fp32 working copy once and
// refills the copy buffer while it walks the working copy.  U is the storage type (the bits
// of a bf16 or an fp32 value); values are widened to fp32 when read.
constexpr int kChunk = 32;

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_one() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

template <typename T> struct Store;
template <> struct Store<float> {
    using type = float;
};
template <> struct Store<__nv_bfloat16> {
    using type = unsigned short;
};

__device__ __forceinline__ float sm1(const float *p) { return *p; }
__device__ __forceinline__ float sm1(const unsigned short *p) { return __uint_as_float(static_cast<uint32_t>(*p) << 16); }
__device__ __forceinline__ float4 sm4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 sm4(const unsigned short *p)
{
    const uint2 x = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(x.x << 16), __uint_as_float(x.x & 0xFFFF0000u), __uint_as_float(x.y << 16),
                       __uint_as_float(x.y & 0xFFFF0000u));
}
// the thread's entries (see ent) of a 64-vector in shared memory
template <int TPR, typename U, int E> __device__ __forceinline__ void smv(const U *vec, int p, float (&o)[E])
{
#pragma unroll
    for (int m = 0; m < E / 4; ++m) {
        const float4 a = sm4(vec + 4 * TPR * m + 4 * p);
        o[4 * m] = a.x, o[4 * m + 1] = a.y, o[4 * m + 2] = a.z, o[4 * m + 3] = a.w;
    }
}

// Copy cnt elements at element offset off of each token t0 .. t0 + nt - 1 (global layout
// base + t stride) into dst[tt][cnt].  cnt * sizeof(U) is a multiple of 16 bytes and every
// source address is 16-byte aligned (token rows are 64 elements apart, off a multiple of 16).
template <typename U>
__device__ __forceinline__ void stage(U *dst, const void *src, int64_t base, int64_t stride, int64_t t0, int nt,
                                      int off, int cnt, int tid)
{
    constexpr int per = 16 / sizeof(U);
    const int pieces = cnt / per;
    const U *g = static_cast<const U *>(src);
    for (int q = tid; q < nt * pieces; q += kThreads) {
        const int tt = q / pieces, x = (q % pieces) * per;
        cp16(dst + tt * cnt + x, g + base + (t0 + tt) * stride + off + x);
    }
}

// a chunk of the row-walking kernels as copied: all 64 channels of v and dy, the CTA's rows
// of r, k, w
template <typename U, int R> struct RowStage {
    U v[kChunk][kN], g[kChunk][kN];
    U r[kChunk][R], k[kChunk][R], w[kChunk][R];
};
// a chunk of the column-walking kernel as copied: all 64 channels of r, k, w, the CTA's
// columns of dy
template <typename U, int R> struct ColStage {
    U r[kChunk][kN], k[kChunk][kN], w[kChunk][kN];
    U g[kChunk][R];
};
// the same in fp32, with bon[t] = sum_i r_t[i] u[i] k_t[i]
template <int R> struct ColWork {
    float r[kChunk][kN], k[kChunk][kN], w[kChunk][kN];
    float g[kChunk][R];
    float bon[kChunk];
};

template <typename U, int R>
__device__ __forceinline__ void issue_rows(RowStage<U, R> &st, const void *r, const void *k, const void *v,
                                           const void *w, const void *dy, int64_t base, int64_t stride, int64_t t0,
                                           int nt, int rg, int tid)
{
    stage(&st.v[0][0], v, base, stride, t0, nt, 0, kN, tid);
    stage(&st.g[0][0], dy, base, stride, t0, nt, 0, kN, tid);
    stage(&st.r[0][0], r, base, stride, t0, nt, R * rg, R, tid);
    stage(&st.k[0][0], k, base, stride, t0, nt, R * rg, R, tid);
    stage(&st.w[0][0], w, base, stride, t0, nt, R * rg, R, tid);
    cp_commit();
}

// widen cnt4 groups of 4 values (x 4 = nt * row length) from src into dst; with dec, form the
// decay from its logit
template <typename U>
__device__ __forceinline__ void widen(float *dst, const U *src, int cnt4, int tid, bool dec)
{
    for (int q = tid; q < cnt4; q += kThreads) {
        float4 x = sm4(src + 4 * q);
        if (dec) x = make_float4(decay(x.x, true), decay(x.y, true), decay(x.z, true), decay(x.w, true));
        *reinterpret_cast<float4 *>(dst + 4 * q) = x;
    }
}

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
    return x;
}

// ------------------------------------------------------------------ forward: dr, du, checkpoints
// CTA (n = b*H + h, row group rg): rows i = R rg .. R rg + R - 1 of S, TPR threads per row.
// Rows of S evolve independently, so the row groups of one head run as separate CTAs.
// Chunks are double-buffered: chunk c + 1 is copied while chunk c is walked.  Checkpoints
// are written row-major (entry i*64 + j of a 64 x 64 block).
template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_forward_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                        const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                        const float *__restrict__ s0, const T *__restrict__ dy, float *__restrict__ dr,
                        float *__restrict__ ckpt, float *__restrict__ du_part, int omega, const int *only,
                        int *status)
{
    using U = typename Store<T>::type;
    constexpr int R = kThreads / TPR, E = kN / TPR;
    extern __shared__ __align__(16) unsigned char smem[];
    RowStage<U, R> *stg = reinterpret_cast<RowStage<U, R> *>(smem);  // [2]
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    if (only && !only[n]) return;
    if (kDebugBounds) {  // every token row of this (b, h) inside [B, T, H, N]
        const int64_t lim = static_cast<int64_t>(gridDim.x) * Tlen * kN, r0 = (b * Tlen * H + h) * kN;
        if (!__syncthreads_and(in_bounds(status, r0, kN, lim) && in_bounds(status, r0 + (Tlen - 1) * H * kN, kN, lim)))
            return;
    }
    const int rg = blockIdx.y, tid = threadIdx.x, p = tid % TPR, il = tid / TPR;
    const int i = R * rg + il;
    const int64_t nblk = (Tlen + kBlock - 1) / kBlock;
    const int64_t nchunks = (Tlen + kChunk - 1) / kChunk;
    const float ui = u[h * kN + i];
    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;

    float S[E];
#pragma unroll
    for (int e = 0; e < E; ++e) S[e] = s0 ? s0[n * kN * kN + i * kN + ent<TPR>(p, e)] : 0.f;

    float du_acc = 0.f;
    issue_rows(stg[0], r, k, v, w, dy, base, stride, 0, static_cast<int>(std::min<int64_t>(kChunk, Tlen)), rg, tid);
    for (int64_t c = 0; c < nchunks; ++c) {
        const int64_t t0 = c * kChunk;
        const int nt = static_cast<int>(std::min<int64_t>(kChunk, Tlen - t0));
        if (c + 1 < nchunks) {
            issue_rows(stg[(c + 1) & 1], r, k, v, w, dy, base, stride, t0 + kChunk,
                       static_cast<int>(std::min<int64_t>(kChunk, Tlen - t0 - kChunk)), rg, tid);
            cp_wait_one();
        } else {
            cp_wait_all();
        }
        __syncthreads();
        const RowStage<U, R> &st = stg[c & 1];
        for (int tt = 0; tt < nt; ++tt) {
            const int64_t t = t0 + tt;
            if (t % kBlock == 0 &&  // checkpoint: the state before this token
                in_bounds(status, (n * nblk + t / kBlock) * (kN * kN) + i * kN, kN, gridDim.x * nblk * kN * kN)) {
                float *cp = ckpt + (n * nblk + t / kBlock) * (kN * kN) + i * kN;
#pragma unroll
                for (int m = 0; m < E / 4; ++m)
                    *reinterpret_cast<float4 *>(cp + ent<TPR>(p, 4 * m)) =
                        make_float4(S[4 * m], S[4 * m + 1], S[4 * m + 2], S[4 * m + 3]);
            }
            float xv[E], xg[E];
            smv<TPR>(st.v[tt], p, xv);
            smv<TPR>(st.g[tt], p, xg);
            const float xr = sm1(&st.r[tt][il]), xk = sm1(&st.k[tt][il]);
            const float xw = decay(sm1(&st.w[tt][il]), omega);
            float sd = 0.f, dot = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) {
                sd = fmaf(S[e], xg[e], sd);
                dot = fmaf(xg[e], xv[e], dot);
                S[e] = fmaf(xw, S[e], xk * xv[e]);
            }
            sd = group_sum<TPR>(sd);
            dot = group_sum<TPR>(dot);
            if (p == 0) dr[base + t * stride + i] = fmaf(ui * xk, dot, sd);
            du_acc = fmaf(xr * xk, dot, du_acc);
        }
        __syncthreads();  // this buffer is refilled for chunk c + 2 next
    }
    if (p == 0) du_part[n * kN + i] = du_acc;
}

// ------------------------------------------------------------------ backward, rows: dk, dw
// Same CTA and thread layout as the forward kernel; chunks (double-buffered) and the tokens
// in them are walked last to first.  For each block of kBlock tokens, the states before
// its tokens are first recomputed from the block's checkpoint into a per-thread
// shared-memory stash.
template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_rows_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                     const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                     const T *__restrict__ dy, const float *__restrict__ dsT, const float *__restrict__ ckpt,
                     float *__restrict__ dk, float *__restrict__ dw, int omega, const int *only, int *status)
{
    using U = typename Store<T>::type;
    constexpr int R = kThreads / TPR, E = kN / TPR, G = E / 4;
    extern __shared__ __align__(16) unsigned char smem[];
    RowStage<U, R> *stg = reinterpret_cast<RowStage<U, R> *>(smem);  // [2]
    float4(*stash)[G][kThreads] = reinterpret_cast<float4(*)[G][kThreads]>(smem + 2 * sizeof(RowStage<U, R>));
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    if (only && !only[n]) return;
    if (kDebugBounds) {  // every token row of this (b, h) inside [B, T, H, N]
        const int64_t lim = static_cast<int64_t>(gridDim.x) * Tlen * kN, r0 = (b * Tlen * H + h) * kN;
        if (!__syncthreads_and(in_bounds(status, r0, kN, lim) && in_bounds(status, r0 + (Tlen - 1) * H * kN, kN, lim)))
            return;
    }
    const int rg = blockIdx.y, tid = threadIdx.x, p = tid % TPR, il = tid / TPR;
    const int i = R * rg + il;
    const int64_t nblk = (Tlen + kBlock - 1) / kBlock;
    const int64_t nchunks = (Tlen + kChunk - 1) / kChunk;
    const float ui = u[h * kN + i];
    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;

    float L[E];
#pragma unroll
    for (int e = 0; e < E; ++e) L[e] = dsT ? dsT[n * kN * kN + i * kN + ent<TPR>(p, e)] : 0.f;

    // this thread's part of a block's checkpoint, loaded one block ahead
    float4 nx[G];
    auto ck = [&](int64_t cb) {
        if (!in_bounds(status, (n * nblk + cb) * (kN * kN) + i * kN, kN, gridDim.x * nblk * kN * kN)) return;
        const float *cp = ckpt + (n * nblk + cb) * (kN * kN) + i * kN;
#pragma unroll
        for (int m = 0; m < G; ++m) nx[m] = *reinterpret_cast<const float4 *>(cp + ent<TPR>(p, 4 * m));
    };
    ck(nblk - 1);
    {
        const int64_t t0 = (nchunks - 1) * kChunk;
        issue_rows(stg[(nchunks - 1) & 1], r, k, v, w, dy, base, stride, t0, static_cast<int>(Tlen - t0), rg, tid);
    }
    for (int64_t c = nchunks - 1; c >= 0; --c) {
        const int64_t t0 = c * kChunk;
        const int nt = static_cast<int>(std::min<int64_t>(kChunk, Tlen - t0));
        if (c > 0) {
            issue_rows(stg[(c - 1) & 1], r, k, v, w, dy, base, stride, t0 - kChunk, kChunk, rg, tid);
            cp_wait_one();
        } else {
            cp_wait_all();
        }
        __syncthreads();
        const RowStage<U, R> &st = stg[c & 1];
        for (int blk = (nt - 1) / kBlock; blk >= 0; --blk) {
            const int64_t cb = t0 / kBlock + blk;  // global block index
            const int tb = kBlock * blk;           // first token of the block within the chunk
            const int tv = nt - tb < kBlock ? nt - tb : kBlock;
            float sv[E];
#pragma unroll
            for (int m = 0; m < G; ++m) {
                sv[4 * m] = nx[m].x, sv[4 * m + 1] = nx[m].y, sv[4 * m + 2] = nx[m].z, sv[4 * m + 3] = nx[m].w;
            }
            if (cb > 0) ck(cb - 1);
#pragma unroll
            for (int tt = 0; tt < kBlock; ++tt) {
                if (tt < tv) {
#pragma unroll
                    for (int m = 0; m < G; ++m)
                        stash[tt][m][tid] = make_float4(sv[4 * m], sv[4 * m + 1], sv[4 * m + 2], sv[4 * m + 3]);
                    if (tt + 1 < tv) {
                        float xv[E];
                        smv<TPR>(st.v[tb + tt], p, xv);
                        const float xk = sm1(&st.k[tb + tt][il]);
                        const float xw = decay(sm1(&st.w[tb + tt][il]), omega);
#pragma unroll
                        for (int e = 0; e < E; ++e) sv[e] = fmaf(xw, sv[e], xk * xv[e]);
                    }
                }
            }
#pragma unroll
            for (int tt = kBlock - 1; tt >= 0; --tt) {
                if (tt < tv) {
                    float sp[E], xv[E], xg[E];
#pragma unroll
                    for (int m = 0; m < G; ++m) {
                        const float4 a = stash[tt][m][tid];
                        sp[4 * m] = a.x, sp[4 * m + 1] = a.y, sp[4 * m + 2] = a.z, sp[4 * m + 3] = a.w;
                    }
                    smv<TPR>(st.v[tb + tt], p, xv);
                    smv<TPR>(st.g[tb + tt], p, xg);
                    const float xr = sm1(&st.r[tb + tt][il]), om = sm1(&st.w[tb + tt][il]);
                    const float xw = decay(om, omega);
                    float dwp = 0.f, dkp = 0.f, dot = 0.f;
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        dwp = fmaf(L[e], sp[e], dwp);
                        dkp = fmaf(L[e], xv[e], dkp);
                        dot = fmaf(xg[e], xv[e], dot);
                        L[e] = fmaf(xw, L[e], xr * xg[e]);
                    }
                    dwp = group_sum<TPR>(dwp);
                    dkp = group_sum<TPR>(dkp);
                    dot = group_sum<TPR>(dot);
                    if (p == 0) {
                        const int64_t o = base + (t0 + tb + tt) * stride + i;
                        dk[o] = fmaf(ui * xr, dot, dkp);
                        // with the logit: dw/domega = -exp(omega) w
                        dw[o] = omega ? dwp * (-expf(om) * xw) : dwp;
                    }
                }
            }
        }
        __syncthreads();  // this buffer is refilled for chunk c - 2 next
    }
}

// ------------------------------------------------------------------ backward, columns: dv, ds0
// CTA (n, column group cg): R = CPT kThreads / TPR columns of the state gradient.  TPR
// threads share a column and each holds E of its rows; a thread serves CPT columns
// (jl + m kThreads / TPR), so every r, k, w value it reads from shared memory feeds CPT
// columns (columns evolve independently).
template <typename T, int TPR, int CPT>
__global__ void __launch_bounds__(kThreads)
wkv6_bwd_cols_kernel(int64_t Tlen, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                     const T *__restrict__ w, const float *__restrict__ u, const T *__restrict__ dy,
                     const float *__restrict__ dsT, float *__restrict__ dv, float *__restrict__ ds0, int omega,
                     const int *only, int *status)
{
    using U = typename Store<T>::type;
    constexpr int S = kThreads / TPR, R = S * CPT, E = kN / TPR;
    extern __shared__ __align__(16) unsigned char smem[];
    ColStage<U, R> &st = *reinterpret_cast<ColStage<U, R> *>(smem);
    ColWork<R> &wk = *reinterpret_cast<ColWork<R> *>(smem + sizeof(ColStage<U, R>));
    const int64_t n = blockIdx.x, b = n / H, h = n % H;
    if (only && !only[n]) return;
    if (kDebugBounds) {  // every token row of this (b, h) inside [B, T, H, N]
        const int64_t lim = static_cast<int64_t>(gridDim.x) * Tlen * kN, r0 = (b * Tlen * H + h) * kN;
        if (!__syncthreads_and(in_bounds(status, r0, kN, lim) && in_bounds(status, r0 + (Tlen - 1) * H * kN, kN, lim)))
            return;
    }
    const int cg = blockIdx.y, tid = threadIdx.x, p = tid % TPR, jl = tid / TPR;
    const int warp = tid / 32, lane = tid % 32;
    const int64_t nchunks = (Tlen + kChunk - 1) / kChunk;
    const int64_t stride = H * kN;
    const int64_t base = (b * Tlen * H + h) * kN;
    float L[CPT][E];
#pragma unroll
    for (int c = 0; c < CPT; ++c)
#pragma unroll
        for (int e = 0; e < E; ++e)
            L[c][e] = dsT ? dsT[n * kN * kN + ent<TPR>(p, e) * kN + R * cg + jl + S * c] : 0.f;
    const float u0 = u[h * kN + 2 * lane], u1 = u[h * kN + 2 * lane + 1];
    auto issue = [&](int64_t t0, int nt) {
        stage(&st.r[0][0], r, base, stride, t0, nt, 0, kN, tid);
        stage(&st.k[0][0], k, base, stride, t0, nt, 0, kN, tid);
        stage(&st.w[0][0], w, base, stride, t0, nt, 0, kN, tid);
        stage(&st.g[0][0], dy, base, stride, t0, nt, R * cg, R, tid);
        cp_commit();
    };
    {
        const int64_t t0 = (nchunks - 1) * kChunk;
        issue(t0, static_cast<int>(Tlen - t0));
    }
    for (int64_t ch = nchunks - 1; ch >= 0; --ch) {
        const int64_t t0 = ch * kChunk;
        const int nt = static_cast<int>(std::min<int64_t>(kChunk, Tlen - t0));
        cp_wait_all();
        __syncthreads();  // chunk ch copied; the previous chunk's working copy no longer read
        widen(&wk.r[0][0], &st.r[0][0], nt * kN / 4, tid, false);
        widen(&wk.k[0][0], &st.k[0][0], nt * kN / 4, tid, false);
        widen(&wk.w[0][0], &st.w[0][0], nt * kN / 4, tid, omega != 0);
        widen(&wk.g[0][0], &st.g[0][0], nt * R / 4, tid, false);
        for (int tt = warp; tt < nt; tt += kThreads / 32) {
            const float q = sm1(&st.r[tt][2 * lane]) * u0 * sm1(&st.k[tt][2 * lane]) +
                            sm1(&st.r[tt][2 * lane + 1]) * u1 * sm1(&st.k[tt][2 * lane + 1]);
            const float sum = warp_sum(q);
            if (lane == 0) wk.bon[tt] = sum;
        }
        __syncthreads();  // working copy ready; the copy buffer is free
        if (ch > 0) issue(t0 - kChunk, kChunk);
        for (int tt = nt - 1; tt >= 0; --tt) {
            float xr[E], xk[E], xw[E];
            smv<TPR>(wk.r[tt], p, xr);
            smv<TPR>(wk.k[tt], p, xk);
            smv<TPR>(wk.w[tt], p, xw);
#pragma unroll
            for (int c = 0; c < CPT; ++c) {
                const float xg = wk.g[tt][jl + S * c];
                float dvp = 0.f;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    dvp = fmaf(L[c][e], xk[e], dvp);
                    L[c][e] = fmaf(xw[e], L[c][e], xr[e] * xg);
                }
                dvp = group_sum<TPR>(dvp);
                if (p == 0) dv[base + (t0 + tt) * stride + R * cg + jl + S * c] = fmaf(wk.bon[tt], xg, dvp);
            }
        }
    }
    if (ds0) {
#pragma unroll
        for (int c = 0; c < CPT; ++c)
#pragma unroll
            for (int e = 0; e < E; ++e) ds0[n * kN * kN + ent<TPR>(p, e) * kN + R * cg + jl + S * c] = L[c][e];
    }
}

// du[h][i] = the sum over batch rows b of the (b, h) sequence's share: du_part[b][h][i] from
// the walks, or, where the chunked path served the sequence (flags given and the sequence's
// flag clear), its chunks' du_item[b][h][c][i].  kDuParts threads per channel each sum a
// fixed share of the terms (chunks c = q mod kDuParts) in order of (b, c), and the shares are
// added in order: the result is deterministic.
constexpr int kDuParts = 16;
__global__ void __launch_bounds__(kN * kDuParts) wkv6_bwd_du_kernel(int64_t B, int64_t H, int64_t nch,
                                                                   const float *__restrict__ du_part,
                                                                   const float *__restrict__ du_item,
                                                                   const int *__restrict__ flags,
                                                                   float *__restrict__ du)
{
    __shared__ float part[kDuParts][kN];
    const int64_t h = blockIdx.x;
    const int i = threadIdx.x % kN, q = threadIdx.x / kN;
    float acc = 0.f;
    for (int64_t b = 0; b < B; ++b) {
        const int64_t n = b * H + h;
        if (!flags || flags[n]) {
            if (q == 0) acc += du_part[n * kN + i];
        } else {
            const float *src = du_item + n * nch * kN + i;
#pragma unroll 4
            for (int64_t c = q; c < nch; c += kDuParts) acc += src[c * kN];
        }
    }
    part[q][i] = acc;
    __syncthreads();
    if (q == 0) {
        float s = part[0][i];
#pragma unroll
        for (int j = 1; j < kDuParts; ++j) s += part[j][i];
        du[h * kN + i] = s;
    }
}

// threads per row (column) of each kernel: the row walk backwards keeps a stash of kBlock
// states per row in shared memory, so it spreads a row over more threads
constexpr int kFwdTPR = 4, kRowsTPR = 8, kColsTPR = 8, kColsCPT = 2;

template <typename T> constexpr int fwd_smem()
{
    return 2 * static_cast<int>(sizeof(RowStage<typename Store<T>::type, kThreads / kFwdTPR>));
}
template <typename T> constexpr int rows_smem()
{
    return 2 * static_cast<int>(sizeof(RowStage<typename Store<T>::type, kThreads / kRowsTPR>)) +
           kBlock * kThreads * (kN / kRowsTPR) * 4;
}
template <typename T> constexpr int cols_smem()
{
    constexpr int R = kThreads / kColsTPR * kColsCPT;
    return static_cast<int>(sizeof(ColStage<typename Store<T>::type, R>) + sizeof(ColWork<R>));
}

template <typename T> cudaError_t configure()
{
    cudaError_t e = cudaFuncSetAttribute(wkv6_bwd_forward_kernel<T, kFwdTPR>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, fwd_smem<T>());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(wkv6_bwd_rows_kernel<T, kRowsTPR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 rows_smem<T>());
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(wkv6_bwd_cols_kernel<T, kColsTPR, kColsCPT>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, cols_smem<T>());
    return e;
}

template <typename T>
cudaError_t launch_all(const Wkv6BwdArgs &a, const BwdLayout &L, const int *only, cudaStream_t s)
{
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            e = configure<T>();
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    const int64_t bh = a.B * a.H;
    unsigned char *ws = static_cast<unsigned char *>(a.workspace);
    float *ckpt = reinterpret_cast<float *>(ws);
    float *du_part = reinterpret_cast<float *>(ws + L.du_part);
    const int om = a.omega ? 1 : 0;
    const unsigned nbh = static_cast<unsigned>(bh);
    const T *r = static_cast<const T *>(a.r), *k = static_cast<const T *>(a.k);
    const T *v = static_cast<const T *>(a.v), *w = static_cast<const T *>(a.w);
    const T *dy = static_cast<const T *>(a.dy);
    // grid: (b, h) x the row (column) groups of a head
    wkv6_bwd_forward_kernel<T, kFwdTPR><<<dim3(nbh, kFwdTPR / 2), kThreads, fwd_smem<T>(), s>>>(
        a.T, a.H, r, k, v, w, a.u, a.s0, dy, a.dr, ckpt, du_part, om, only, a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv6_bwd_rows_kernel<T, kRowsTPR><<<dim3(nbh, kRowsTPR / 2), kThreads, rows_smem<T>(), s>>>(
        a.T, a.H, r, k, v, w, a.u, dy, a.dsT, ckpt, a.dk, a.dw, om, only, a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    wkv6_bwd_cols_kernel<T, kColsTPR, kColsCPT><<<dim3(nbh, kN / (kThreads / kColsTPR * kColsCPT)), kThreads,
                                                   cols_smem<T>(), s>>>(
        a.T, a.H, r, k, w, a.u, dy, a.dsT, a.dv, a.ds0, om, only, a.status);
    return cudaGetLastError();
}

}  // namespace

BwdLayout wkv6_backward_layout(int64_t B, int64_t T, int64_t H)
{
    const size_t bh = static_cast<size_t>(B * H);
    const size_t nblk = static_cast<size_t>((T + kBlock - 1) / kBlock);
    const size_t nch = static_cast<size_t>((T + 63) / 64);
    BwdLayout L{};
    L.nch = static_cast<int64_t>(nch);
    const size_t walks = bh * nblk * kN * kN * sizeof(float);  // fp32 checkpoints every kBlock tokens
    L.sck = 0;                                                 // bf16 [bh][nch + 1][64][64]
    L.dsck = L.sck + bh * (nch + 1) * kN * kN * 2;             // bf16 [bh][nch][64][64]
    L.rowdot = L.dsck + bh * nch * kN * kN * 2;                // fp32 [bh][nch][64]
    const size_t chunked = L.rowdot + bh * nch * kN * sizeof(float);
    L.du_part = std::max(walks, chunked);                      // fp32 [bh][64]
    L.du_item = L.du_part + bh * kN * sizeof(float);           // fp32 [bh][nch][64]
    L.flags = L.du_item + bh * nch * kN * sizeof(float);       // int [bh]
    L.total = L.flags + ((bh * sizeof(int) + 15) & ~static_cast<size_t>(15));
    return L;
}

size_t wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H) { return wkv6_backward_layout(B, T, H).total; }

cudaError_t wkv6_backward_walks_launch(const Wkv6BwdArgs &a, const BwdLayout &L, const int *only, cudaStream_t s)
{
    return a.bf16 ? launch_all<__nv_bfloat16>(a, L, only, s) : launch_all<float>(a, L, only, s);
}

cudaError_t wkv6_backward_launch(const Wkv6BwdArgs &a, cudaStream_t s)
{
    if (a.B * a.H == 0 || a.T == 0) return cudaSuccess;
    if (a.B * a.H > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const BwdLayout L = wkv6_backward_layout(a.B, a.T, a.H);
    unsigned char *ws = static_cast<unsigned char *>(a.workspace);
    const int *flags = nullptr;
    cudaError_t e;
    if (a.chunked && a.bf16) {
        // the tensor-core path; the sequences it flags (decay too fast for its chunk algebra)
        // are then served by the exact walks
        e = wkv6_backward_tc_launch(a, L, s);
        if (e != cudaSuccess) return e;
        flags = reinterpret_cast<const int *>(ws + L.flags);
    }
    e = wkv6_backward_walks_launch(a, L, flags, s);
    if (e != cudaSuccess) return e;
    wkv6_bwd_du_kernel<<<static_cast<unsigned>(a.H), kN * kDuParts, 0, s>>>(
        a.B, a.H, L.nch, reinterpret_cast<const float *>(ws + L.du_part),
        reinterpret_cast<const float *>(ws + L.du_item), flags, a.du);
    return cudaGetLastError();
}

}  // namespace wkv
