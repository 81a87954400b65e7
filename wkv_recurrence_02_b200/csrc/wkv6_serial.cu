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
// Both kernels can take the decay as its logit omega_t and form w_t = exp(-exp(omega_t)) as
// they load it.
#include "wkv_internal.cuh"

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

cudaError_t wkv6_decode_launch(const Wkv6Args &a, cudaStream_t s)
{
    if (a.T != 1) return wkv6_serial_launch(a, s);
    const int64_t blocks = a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
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
