// wkv6_serial.cu -- Eagle/Finch WKV-6 evaluated token by token on CUDA cores (fp32).
//
// Source: "RWKV-5/6 (Eagle and Finch)", section 4.1.2 (Eagle time mixing: state s is a
// sum of k^T v, each key channel decayed by its w every step; gain u on the current
// token's k^T v; receptance r applied like a query) and section 4.2.2 (Finch: w_t per
// token); section 4 fixes row vectors with matrices acting on the right, so the state
// is N x N with row i = key channel and column j = value channel.  RNN-mode decoding
// with constant memory per token is the RWKV-4 paper's section "类 RNN 的序列解码".
//
// Two kernels:
//  * wkv6_serial_kernel -- any T, fp32 or bf16 inputs.  One CTA per (b, h), one thread
//    per value column j holding S[:, j] (64 fp32) in registers, so the output
//    o_t[j] = sum_i r_t[i] (S[i][j] + u[i] k_t[i] v_t[j]) needs no cross-thread
//    reduction.  r_t, k_t, w_t are broadcast through double-buffered shared memory and
//    the next token's inputs are prefetched into registers while the current one is
//    processed.  This is the fp32-accuracy path (tensor cores cannot meet fp32
//    tolerances) and the reference path the chunked kernel is tested against.
//  * wkv6_decode_kernel -- T == 1: one (b, h) per 256-thread CTA; thread (ig, j4) owns
//    rows 4ig..4ig+3 x columns 4j4..4j4+3 of S and moves them with 16-byte loads and
//    stores, so the 2 x 16 KB state stream per head is fully coalesced.  Partial
//    outputs are reduced over the 16 row groups through shared memory.  With a gate g the
//    64 outputs of the head go through the fused LayerNorm + SiLU gate before the store.
//    It serves T == 1 calls with the fused output stage or without an initial state.
//  * wkv6_decode_stream_kernel -- T == 1 with an initial state: the same update by
//    persistent CTAs that stream the heads' states through a ring of bulk copies.
// Both kernels can take the decay as its logit omega_t and form w_t = exp(-exp(omega_t)) as
// they load it.
#include "tc_common.cuh"

#include <algorithm>

namespace wkv {
namespace {

constexpr int kN = 64;

template <typename T> __device__ __forceinline__ float ld(const T *p);
template <> __device__ __forceinline__ float ld<float>(const float *p) { return __ldg(p); }
template <> __device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    return __bfloat162float(*p);
}
template <typename T> __device__ __forceinline__ void st(T *p, float x);
template <> __device__ __forceinline__ void st<float>(float *p, float x) { *p = x; }
template <> __device__ __forceinline__ void st<__nv_bfloat16>(__nv_bfloat16 *p, float x)
{
    *p = __float2bfloat16_rn(x);
}

// Decay from its logit, w = exp(-exp(omega)) (section 4.1.2), with the accurate exponential:
// omega = -inf gives 1, +inf gives 0.
__device__ __forceinline__ float decay_of_logit(float om) { return expf(-expf(om)); }

template <typename T>
__global__ void __launch_bounds__(kN)
wkv6_serial_kernel(int64_t T_len, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                   const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                   const float *s0, T *__restrict__ y, float *sT, int omega, int *status)
{
    __shared__ __align__(16) float sr[2][kN], sk[2][kN], sw[2][kN];
    __shared__ __align__(16) float su[kN];

    const int64_t n = blockIdx.x;  // b * H + h
    const int64_t b = n / H, h = n % H;
    const int j = threadIdx.x;
    if (kDebugBounds) {  // every token row of this (b, h) inside [B, T, H, N]; u of the head
        const int64_t lim = static_cast<int64_t>(gridDim.x) * T_len * kN;
        const int64_t b0 = (b * T_len * H + h) * kN + j;
        const bool ok = in_bounds(status, b0, 1, lim) && in_bounds(status, b0 + (T_len - 1) * H * kN, 1, lim) &&
                        in_bounds(status, h * kN + j, 1, H * kN);
        if (!__syncthreads_and(ok)) return;
    }

    float S[kN];
    const float *s0p = s0 ? s0 + n * kN * kN : nullptr;
#pragma unroll
    for (int i = 0; i < kN; ++i) S[i] = s0p ? s0p[i * kN + j] : 0.f;
    su[j] = u[h * kN + j];

    const int64_t stride = H * kN;
    const int64_t base = (b * T_len * H + h) * kN + j;
    float rn = ld(r + base), kn = ld(k + base), vn = ld(v + base), wn = ld(w + base);

    for (int64_t t = 0; t < T_len; ++t) {
        const int buf = static_cast<int>(t & 1);
        sr[buf][j] = rn;
        sk[buf][j] = kn;
        sw[buf][j] = omega ? decay_of_logit(wn) : wn;
        const float vj = vn;
        __syncthreads();
        if (t + 1 < T_len) {
            const int64_t o = base + (t + 1) * stride;
            rn = ld(r + o);
            kn = ld(k + o);
            vn = ld(v + o);
            wn = ld(w + o);
        }
        const float4 *r4 = reinterpret_cast<const float4 *>(sr[buf]);
        const float4 *k4 = reinterpret_cast<const float4 *>(sk[buf]);
        const float4 *w4 = reinterpret_cast<const float4 *>(sw[buf]);
        const float4 *u4 = reinterpret_cast<const float4 *>(su);
        float acc = 0.f, bonus = 0.f;
#pragma unroll
        for (int i4 = 0; i4 < kN / 4; ++i4) {
            const float4 rr = r4[i4], kk = k4[i4], uu = u4[i4];
            acc = fmaf(rr.x, S[4 * i4 + 0], acc);
            acc = fmaf(rr.y, S[4 * i4 + 1], acc);
            acc = fmaf(rr.z, S[4 * i4 + 2], acc);
            acc = fmaf(rr.w, S[4 * i4 + 3], acc);
            bonus = fmaf(rr.x * uu.x, kk.x, bonus);
            bonus = fmaf(rr.y * uu.y, kk.y, bonus);
            bonus = fmaf(rr.z * uu.z, kk.z, bonus);
            bonus = fmaf(rr.w * uu.w, kk.w, bonus);
        }
        st(y + base + t * stride, fmaf(bonus, vj, acc));
#pragma unroll
        for (int i4 = 0; i4 < kN / 4; ++i4) {
            const float4 kk = k4[i4], ww = w4[i4];
            S[4 * i4 + 0] = fmaf(ww.x, S[4 * i4 + 0], kk.x * vj);
            S[4 * i4 + 1] = fmaf(ww.y, S[4 * i4 + 1], kk.y * vj);
            S[4 * i4 + 2] = fmaf(ww.z, S[4 * i4 + 2], kk.z * vj);
            S[4 * i4 + 3] = fmaf(ww.w, S[4 * i4 + 3], kk.w * vj);
        }
    }
    if (sT) {
        float *sp = sT + n * kN * kN;
#pragma unroll
        for (int i = 0; i < kN; ++i) sp[i * kN + j] = S[i];
    }
}

// Four consecutive channels as fp32.
template <typename T> __device__ __forceinline__ float4 ld4(const T *p);
template <> __device__ __forceinline__ float4 ld4<float>(const float *p)
{
    return __ldg(reinterpret_cast<const float4 *>(p));
}
template <> __device__ __forceinline__ float4 ld4<__nv_bfloat16>(const __nv_bfloat16 *p)
{
    const uint2 raw = __ldg(reinterpret_cast<const uint2 *>(p));
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.x));
    const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&raw.y));
    return make_float4(a.x, a.y, c.x, c.y);
}

__device__ __forceinline__ float comp(const float4 &x, int m)
{
    return m == 0 ? x.x : (m == 1 ? x.y : (m == 2 ? x.z : x.w));
}

template <typename T>
__global__ void __launch_bounds__(256)
wkv6_decode_kernel(int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                   const T *__restrict__ v, const T *__restrict__ w,
                   const float *__restrict__ u, const float *s0, T *__restrict__ y, float *sT,
                   const T *__restrict__ g, const float *__restrict__ ln_w, const float *__restrict__ ln_b,
                   float eps, int omega, int *status)
{
    __shared__ __align__(16) float red[16][kN];
    __shared__ float bred[16];
    __shared__ float stat[2][2];

    const int64_t n = blockIdx.x;  // b * H + h; with T == 1 the token row is n * N
    const int64_t h = n % H;
    const int tid = threadIdx.x, ig = tid >> 4, j4 = tid & 15;
    const int64_t vbase = n * kN;
    if (kDebugBounds) {  // the token row, the state block and u of this thread
        const int64_t nall = gridDim.x;
        const bool ok = in_bounds(status, vbase + 4 * ig, 4, nall * kN) &&
                        in_bounds(status, vbase + 4 * j4, 4, nall * kN) &&
                        in_bounds(status, n * kN * kN + (4 * ig + 3) * kN + 4 * j4, 4, nall * kN * kN) &&
                        in_bounds(status, h * kN + 4 * ig, 4, H * kN);
        if (!__syncthreads_and(ok)) return;
    }

    const float4 rr = ld4(r + vbase + 4 * ig);
    const float4 kk = ld4(k + vbase + 4 * ig);
    float4 ww = ld4(w + vbase + 4 * ig);
    if (omega)
        ww = make_float4(decay_of_logit(ww.x), decay_of_logit(ww.y), decay_of_logit(ww.z), decay_of_logit(ww.w));
    const float4 uu = __ldg(reinterpret_cast<const float4 *>(u + h * kN + 4 * ig));
    const float4 vv = ld4(v + vbase + 4 * j4);

    float4 Srow[4];
    const int64_t sbase = n * kN * kN + (4 * ig) * kN + 4 * j4;
#pragma unroll
    for (int m = 0; m < 4; ++m)
        Srow[m] = s0 ? *reinterpret_cast<const float4 *>(s0 + sbase + m * kN)
                     : make_float4(0.f, 0.f, 0.f, 0.f);

    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float bonus = 0.f;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const float ri = comp(rr, m), ki = comp(kk, m), wi = comp(ww, m);
        o.x = fmaf(ri, Srow[m].x, o.x);
        o.y = fmaf(ri, Srow[m].y, o.y);
        o.z = fmaf(ri, Srow[m].z, o.z);
        o.w = fmaf(ri, Srow[m].w, o.w);
        bonus = fmaf(ri * comp(uu, m), ki, bonus);
        Srow[m].x = fmaf(wi, Srow[m].x, ki * vv.x);
        Srow[m].y = fmaf(wi, Srow[m].y, ki * vv.y);
        Srow[m].z = fmaf(wi, Srow[m].z, ki * vv.z);
        Srow[m].w = fmaf(wi, Srow[m].w, ki * vv.w);
    }
    if (sT) {
#pragma unroll
        for (int m = 0; m < 4; ++m) *reinterpret_cast<float4 *>(sT + sbase + m * kN) = Srow[m];
    }
    *reinterpret_cast<float4 *>(&red[ig][4 * j4]) = o;
    if (j4 == 0) bred[ig] = bonus;
    __syncthreads();
    if (tid < kN) {
        float acc = 0.f, bsum = 0.f;
#pragma unroll
        for (int rg = 0; rg < 16; ++rg) {
            acc += red[rg][tid];
            bsum += bred[rg];
        }
        float o = fmaf(bsum, ld(v + vbase + tid), acc);
        if (g) {
            // fused output stage: LayerNorm over the head's 64 outputs (two warps), SiLU gate
            float s = o;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
            if ((tid & 31) == 0) stat[0][tid >> 5] = s;
            asm volatile("bar.sync 1, 64;" ::: "memory");
            const float mean = (stat[0][0] + stat[0][1]) * (1.f / kN);
            const float d = o - mean;
            float q = d * d;
#pragma unroll
            for (int m = 16; m >= 1; m >>= 1) q += __shfl_xor_sync(0xffffffffu, q, m);
            if ((tid & 31) == 0) stat[1][tid >> 5] = q;
            asm volatile("bar.sync 1, 64;" ::: "memory");
            const float rstd = rsqrtf((stat[1][0] + stat[1][1]) * (1.f / kN) + eps);
            const float gv = ld(g + vbase + tid);
            const float gate = __fdividef(gv, 1.f + __expf(-gv));  // SiLU, fast intrinsics
            o = gate * fmaf(ln_w[h * kN + tid] * d, rstd, ln_b[h * kN + tid]);
        }
        st(y + vbase + tid, o);
    }
}

// ------------------------------------------------------------ streaming decode (T == 1)
// Persistent CTAs of 256 threads, four per SM, each walking heads n = blockIdx.x + i gridDim.x
// through a 3-stage ring: the head's 16 KB state and its r, k, w, v vectors arrive by bulk
// copies (mbarrier), the update is made in shared memory by the same 4 x 4 blocks as the
// kernel above, and the new state leaves by a bulk store.  Two heads' copies stay in flight
// while one is updated (about 130 KB per SM), so the state stream does not stall between
// heads.  The stage of head i - 1 is refilled with head i + 2 once head i - 1's store has read
// it.  Used for every T == 1 call with an initial state and no fused output stage.
constexpr int kDStages = 3;
constexpr int kDThreads = 256;
template <typename T> constexpr int dstage_bytes() { return kN * kN * 4 + 4 * kN * static_cast<int>(sizeof(T)); }
template <typename T> constexpr int decode_stream_smem()
{
    return kDStages * dstage_bytes<T>() + 16 * kN * 4 + 16 * 4 + 8 * kDStages + 128;
}

// Plain load of an element held in shared memory (ld() above is for global memory: its fp32
// form is a read-only global load, which must not be given a shared-memory address).
template <typename T> __device__ __forceinline__ float sld(const T *p);
template <> __device__ __forceinline__ float sld<float>(const float *p) { return *p; }
template <> __device__ __forceinline__ float sld<__nv_bfloat16>(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
// four consecutive values from shared memory in one access (p aligned to 4 elements)
template <typename T> __device__ __forceinline__ void sld4(const T *p, float (&x)[4]);
template <> __device__ __forceinline__ void sld4<float>(const float *p, float (&x)[4])
{
    const float4 q = *reinterpret_cast<const float4 *>(p);
    x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
}
template <> __device__ __forceinline__ void sld4<__nv_bfloat16>(const __nv_bfloat16 *p, float (&x)[4])
{
    const uint2 q = *reinterpret_cast<const uint2 *>(p);
    x[0] = __uint_as_float(q.x << 16), x[1] = __uint_as_float(q.x & 0xFFFF0000u);
    x[2] = __uint_as_float(q.y << 16), x[3] = __uint_as_float(q.y & 0xFFFF0000u);
}

template <typename T>
__global__ void __launch_bounds__(kDThreads)
wkv6_decode_stream_kernel(int64_t BH, int64_t H, const T *__restrict__ r, const T *__restrict__ k,
                          const T *__restrict__ v, const T *__restrict__ w, const float *__restrict__ u,
                          const float *s0, T *__restrict__ y, float *sT, int omega, int *status, uint32_t limit)
{
    extern __shared__ unsigned char smem_raw[];
    // aligned by an offset on the __shared__ array itself (not through an integer), so the
    // compiler keeps the shared state space: its accesses are shared loads and stores, which it
    // may reorder freely around global ones
    unsigned char *sm = smem_raw + ((128u - (tc::smem_u32(smem_raw) & 127u)) & 127u);
    constexpr int SB = dstage_bytes<T>();
    // per-warp partial sums of y and of the bonus, double-buffered by head parity:
    // [parity][warp][64] and [parity][warp] (the same 16 x 64 + 16 floats as one buffer of
    // per-row-group sums)
    float(*red)[8][kN] = reinterpret_cast<float(*)[8][kN]>(sm + kDStages * SB);
    float(*bred)[8] = reinterpret_cast<float(*)[8]>(sm + kDStages * SB + 16 * kN * 4);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kDStages * SB + 16 * kN * 4 + 16 * 4);
    const uint32_t bar0 = tc::smem_u32(&bars[0]);
    const int tid = threadIdx.x, ig = tid >> 4, j4 = tid & 15;
    const int64_t count = (BH - blockIdx.x + gridDim.x - 1) / gridDim.x;  // heads of this CTA

    if (tid == 0) {
        for (int s = 0; s < kDStages; ++s) tc::bar_init(bar0 + 8 * s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    auto issue = [&](int64_t i) {  // one thread: the copies of this CTA's i-th head
        const int64_t n = blockIdx.x + i * gridDim.x;
        const int s = static_cast<int>(i % kDStages);
        unsigned char *stg = sm + s * SB;
        const uint32_t bar = bar0 + 8 * s;
        if (!in_bounds(status, n * kN * kN, kN * kN, BH * kN * kN) || !in_bounds(status, n * kN, kN, BH * kN)) return;
        tc::bar_expect_tx(bar, SB);
        constexpr uint32_t VB = kN * sizeof(T);
        tc::bulk_load(tc::smem_u32(stg), s0 + n * kN * kN, kN * kN * 4, bar);
        tc::bulk_load(tc::smem_u32(stg + kN * kN * 4), r + n * kN, VB, bar);
        tc::bulk_load(tc::smem_u32(stg + kN * kN * 4 + VB), k + n * kN, VB, bar);
        tc::bulk_load(tc::smem_u32(stg + kN * kN * 4 + 2 * VB), w + n * kN, VB, bar);
        tc::bulk_load(tc::smem_u32(stg + kN * kN * 4 + 3 * VB), v + n * kN, VB, bar);
    };
    if (tid == 0)
        for (int64_t i = 0; i < kDStages && i < count; ++i) issue(i);

    int abort = 0;
    for (int64_t i = 0; i < count; ++i) {
        const int64_t n = blockIdx.x + i * gridDim.x, h = n % H;
        const int s = static_cast<int>(i % kDStages);
        unsigned char *stg = sm + s * SB;
        float *S = reinterpret_cast<float *>(stg);
        const T *vr = reinterpret_cast<const T *>(stg + kN * kN * 4);
        const T *vk = vr + kN, *vw = vr + 2 * kN, *vv = vr + 3 * kN;
        // each thread waits for the stage itself; the expiry vote is taken at the barrier below
        const int ok = tc::bar_wait(bar0 + 8 * s, static_cast<uint32_t>((i / kDStages) & 1), limit);
        float rr[4], kk[4], ww[4], uu[4], vj[4];
        sld4(vr + 4 * ig, rr);
        sld4(vk + 4 * ig, kk);
        sld4(vw + 4 * ig, ww);
        sld4(vv + 4 * j4, vj);
        {
            const float4 u4 = __ldg(reinterpret_cast<const float4 *>(u + h * kN + 4 * ig));  // global
            uu[0] = u4.x, uu[1] = u4.y, uu[2] = u4.z, uu[3] = u4.w;
        }
        if (omega) {
#pragma unroll
            for (int m = 0; m < 4; ++m) ww[m] = decay_of_logit(ww[m]);
        }
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        float bonus = 0.f;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float4 *row = reinterpret_cast<float4 *>(S + (4 * ig + m) * kN + 4 * j4);
            float4 x = *row;
            o[0] = fmaf(rr[m], x.x, o[0]);
            o[1] = fmaf(rr[m], x.y, o[1]);
            o[2] = fmaf(rr[m], x.z, o[2]);
            o[3] = fmaf(rr[m], x.w, o[3]);
            bonus = fmaf(rr[m] * uu[m], kk[m], bonus);
            x.x = fmaf(ww[m], x.x, kk[m] * vj[0]);
            x.y = fmaf(ww[m], x.y, kk[m] * vj[1]);
            x.z = fmaf(ww[m], x.z, kk[m] * vj[2]);
            x.w = fmaf(ww[m], x.w, kk[m] * vj[3]);
            *row = x;
        }
        // the warp's two row groups (lanes l and l ^ 16) summed first
#pragma unroll
        for (int q = 0; q < 4; ++q) o[q] += __shfl_xor_sync(0xffffffffu, o[q], 16);
        bonus += __shfl_xor_sync(0xffffffffu, bonus, 16);
        const int pb = static_cast<int>(i & 1), wp = tid >> 5;
        if ((tid & 31) < 16) *reinterpret_cast<float4 *>(&red[pb][wp][4 * j4]) = make_float4(o[0], o[1], o[2], o[3]);
        if ((tid & 31) == 0) bred[pb][wp] = bonus;
        tc::fence_async_smem();  // the new state is read by the bulk store (async proxy)
        if (__syncthreads_or(!ok)) {  // the one barrier of a head; a stage wait that ran out ends here
            abort = 1;
            break;
        }
        if (tid == 0 && sT) {
            if (in_bounds(status, n * kN * kN, kN * kN, BH * kN * kN)) tc::bulk_store(sT + n * kN * kN, tc::smem_u32(stg), kN * kN * 4);
            tc::bulk_commit();
        }
        if (tid < kN) {
            float acc = 0.f, bsum = 0.f;
#pragma unroll
            for (int wq = 0; wq < 8; ++wq) {
                acc += red[pb][wq][tid];
                bsum += bred[pb][wq];
            }
            st<T>(y + n * kN + tid, fmaf(bsum, sld(vv + tid), acc));
        }
        // the stage of head i - 1 takes head i + 2 once that head's store has read it (every
        // thread is past head i - 1: the barrier above)
        if (tid == 0 && i >= 1 && i + 2 < count) {
            if (sT) tc::bulk_wait_read<1>();
            issue(i + 2);
        }
        // this head's partial sums are written again two heads on, after the next head's
        // barrier, which every reader of them reaches after reading them
    }
    if (abort) {
        record_status(status, kStatusTimeout);
        if (tid == 0)  // bounded: the copies in flight land before the CTA exits
            for (int64_t i = 0; i < count && i < kDStages + 2; ++i)
                tc::bar_wait(bar0 + 8 * static_cast<int>(i % kDStages), static_cast<uint32_t>((i / kDStages) & 1), limit);
    }
    if (tid == 0) tc::bulk_wait_all();
}

}  // namespace

cudaError_t wkv6_serial_launch(const Wkv6Args &a, cudaStream_t s)
{
    const int64_t blocks = a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (a.bf16) {
        using T = __nv_bfloat16;
        wkv6_serial_kernel<T><<<static_cast<unsigned>(blocks), kN, 0, s>>>(
            a.T, a.H, static_cast<const T *>(a.r), static_cast<const T *>(a.k),
            static_cast<const T *>(a.v), static_cast<const T *>(a.w), a.u, a.s0,
            static_cast<T *>(a.y), a.sT, a.omega ? 1 : 0, a.status);
    } else {
        wkv6_serial_kernel<float><<<static_cast<unsigned>(blocks), kN, 0, s>>>(
            a.T, a.H, static_cast<const float *>(a.r), static_cast<const float *>(a.k),
            static_cast<const float *>(a.v), static_cast<const float *>(a.w), a.u, a.s0,
            static_cast<float *>(a.y), a.sT, a.omega ? 1 : 0, a.status);
    }
    return cudaGetLastError();
}

namespace {
template <typename T> cudaError_t launch_decode_stream(const Wkv6Args &a, cudaStream_t s)
{
    static bool done[64] = {};
    int dev = 0, sms = 148;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!done[dev]) {  // racing first calls set the same attribute: harmless
        e = cudaFuncSetAttribute(wkv6_decode_stream_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 decode_stream_smem<T>());
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) sms = 148;
    int per_sm = 0;  // resident CTAs per SM (shared memory bound): the grid stays one wave
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, wkv6_decode_stream_kernel<T>, kDThreads,
                                                      decode_stream_smem<T>());
    if (e != cudaSuccess) return e;
    const int64_t bh = a.B * a.H;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>(bh, static_cast<int64_t>(std::max(per_sm, 1)) * sms));
    wkv6_decode_stream_kernel<T><<<grid, kDThreads, decode_stream_smem<T>(), s>>>(
        bh, a.H, static_cast<const T *>(a.r), static_cast<const T *>(a.k), static_cast<const T *>(a.v),
        static_cast<const T *>(a.w), a.u, a.s0, static_cast<T *>(a.y), a.sT, a.omega ? 1 : 0, a.status, 100000u);
    return cudaGetLastError();
}
}  // namespace

cudaError_t wkv6_decode_launch(const Wkv6Args &a, cudaStream_t s)
{
    if (a.T != 1) return wkv6_serial_launch(a, s);
    const int64_t blocks = a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    // the streaming kernel: an initial state to stream, no fused output stage
    if (a.s0 && !a.g)
        return a.bf16 ? launch_decode_stream<__nv_bfloat16>(a, s) : launch_decode_stream<float>(a, s);
    if (a.bf16) {
        using T = __nv_bfloat16;
        wkv6_decode_kernel<T><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            a.H, static_cast<const T *>(a.r), static_cast<const T *>(a.k),
            static_cast<const T *>(a.v), static_cast<const T *>(a.w), a.u, a.s0,
            static_cast<T *>(a.y), a.sT, static_cast<const T *>(a.g), a.ln_w, a.ln_b, a.eps, a.omega ? 1 : 0,
            a.status);
    } else {
        wkv6_decode_kernel<float><<<static_cast<unsigned>(blocks), 256, 0, s>>>(
            a.H, static_cast<const float *>(a.r), static_cast<const float *>(a.k),
            static_cast<const float *>(a.v), static_cast<const float *>(a.w), a.u, a.s0,
            static_cast<float *>(a.y), a.sT, nullptr, nullptr, nullptr, 0.f, a.omega ? 1 : 0, a.status);
    }
    return cudaGetLastError();
}

}  // namespace wkv
