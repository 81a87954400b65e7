// wkv4_scan.cu -- RWKV-4 WKV on B200: a T-segmented running-maximum scan.
//
// Source: "RWKV: Reinventing RNNs for the Transformer Era" (Chinese translation),
// eq. 14 as referenced in the temporal-structure section (time decay e^{-w}, bonus
// e^{u}), evaluated with the single-step time-dependent softmax of the gradient-
// stability section; the parallelisation section states that this update is a serial
// scan of cost O(BTd).
//
// Per (batch row, channel) the past sums are carried as (a, b, p): numerator a 2^p and
// denominator b 2^p, with p kept in log2 units so every exponential is one ex2.  The
// per-step update is associative once a block of n steps is summarised by its local
// state and its total decay n*w, so T is cut into 32 segments per tile:
//   pass 1  each lane scans its own segment from the empty state;
//   scan    a 5-step warp shuffle scan combines segment summaries across lanes,
//           and the carry from earlier tiles (or s0) is folded in;
//   pass 2  each lane re-walks its segment from its exact incoming state, producing y.
//
// Layout: one CTA = one batch row x 16 channels; warp = channel pair (2 channels per
// lane), lane = segment.  k and v of a tile (32*L tokens x 16 channels) are staged in
// shared memory as 2-channel words in a [pair][segment][L+1] layout: the +1 pad makes
// lane-strided reads conflict-free, and row-contiguous fills stay coalesced from HBM.
// y overwrites k's words in place and is written back with the same coalesced pattern.
#include "wkv_internal.cuh"

namespace wkv {
namespace {

constexpr int kSegs = 32;          // segments per tile (= lanes)
constexpr int kCh = 16;            // channels per CTA
constexpr int kPairs = kCh / 2;    // warps per CTA
constexpr int kThreads = kPairs * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kPEmpty = -1e30f;  // exponent of an empty state (finite: empty+empty stays 0)

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

struct St {
    float a, b, p;
};

// State `e` (earlier), followed by a block whose local state is `l` and whose total
// log2-decay is nw (= its length times w in log2 units).
__device__ __forceinline__ St combine(St e, St l, float nw)
{
    const float pe = e.p - nw;
    const float q = fmaxf(pe, l.p);
    const float fe = ex2(pe - q), fl = ex2(l.p - q);
    return {fmaf(e.a, fe, l.a * fl), fmaf(e.b, fe, l.b * fl), q};
}

// One token into the state: decay the past by 2^{-w2}, add 2^{k2} (v | 1).
__device__ __forceinline__ void update(St &s, float k2, float v, float w2)
{
    const float d = (s.p - w2) - k2;
    const float e = ex2(-fabsf(d));
    const bool past = d >= 0.f;
    const float fs = past ? 1.f : e;
    const float fk = past ? e : 1.f;
    s.a = fmaf(fs, s.a, fk * v);
    s.b = fmaf(fs, s.b, fk);
    s.p = past ? s.p - w2 : k2;
}

// Output of one token: the carried sums plus the bonus term 2^{u2 + k2} v.
__device__ __forceinline__ float output(const St &s, float k2, float v, float u2)
{
    const float d = s.p - (u2 + k2);
    const float e = ex2(-fabsf(d));
    const bool past = d >= 0.f;
    const float fs = past ? 1.f : e;
    const float fk = past ? e : 1.f;
    return __fdividef(fmaf(fs, s.a, fk * v), fmaf(fs, s.b, fk));
}

__device__ __forceinline__ St shfl_up(St s, int off)
{
    return {__shfl_up_sync(0xffffffffu, s.a, off), __shfl_up_sync(0xffffffffu, s.b, off),
            __shfl_up_sync(0xffffffffu, s.p, off)};
}

__device__ __forceinline__ St shfl_idx(St s, int lane)
{
    return {__shfl_sync(0xffffffffu, s.a, lane), __shfl_sync(0xffffffffu, s.b, lane),
            __shfl_sync(0xffffffffu, s.p, lane)};
}

// 2-channel word types and conversions.
template <typename T> struct Word;
template <> struct Word<float> {
    using type = float2;
    __device__ static float2 to_f2(float2 x) { return x; }
    __device__ static float2 from_f2(float2 x) { return x; }
};
template <> struct Word<__nv_bfloat16> {
    using type = __nv_bfloat162;
    __device__ static float2 to_f2(__nv_bfloat162 x) { return __bfloat1622float2(x); }
    __device__ static __nv_bfloat162 from_f2(float2 x) { return __float22bfloat162_rn(x); }
};

template <typename T> struct Elem;
template <> struct Elem<float> {
    __device__ static float get(const float *p) { return *p; }
    __device__ static void put(float *p, float x) { *p = x; }
};
template <> struct Elem<__nv_bfloat16> {
    __device__ static float get(const __nv_bfloat16 *p) { return __bfloat162float(*p); }
    __device__ static void put(__nv_bfloat16 *p, float x) { *p = __float2bfloat16_rn(x); }
};

// Moves one tile between global [rows x 16 channels] and the staged word layout.
// TO_SMEM: global -> smem; otherwise smem -> global.  16-byte vectors when the whole
// channel block is in range and C keeps rows 16-byte aligned; element-wise otherwise.
template <typename T, int L, bool TO_SMEM>
__device__ __forceinline__ void move_tile(typename Word<T>::type *sw, T *g, int64_t row0,
                                          int nt, int64_t C, int c0, bool vec)
{
    using W = typename Word<T>::type;
    constexpr int kWordsPerVec = 16 / sizeof(W);     // 4 (bf16x2) or 2 (float2)
    constexpr int kVecPerRow = kPairs / kWordsPerVec; // 2 or 4
    if (vec) {
        for (int idx = threadIdx.x; idx < nt * kVecPerRow; idx += kThreads) {
            const int r = idx / kVecPerRow, q = idx % kVecPerRow;
            const int seg = r / L, j = r % L;
            T *gp = g + (row0 + r) * C + c0 + q * kWordsPerVec * 2;
            union {
                uint4 u;
                W w[kWordsPerVec];
            } buf;
            if (TO_SMEM) {
                buf.u = __ldg(reinterpret_cast<const uint4 *>(gp));
#pragma unroll
                for (int m = 0; m < kWordsPerVec; ++m)
                    sw[((q * kWordsPerVec + m) * kSegs + seg) * (L + 1) + j] = buf.w[m];
            } else {
#pragma unroll
                for (int m = 0; m < kWordsPerVec; ++m)
                    buf.w[m] = sw[((q * kWordsPerVec + m) * kSegs + seg) * (L + 1) + j];
                *reinterpret_cast<uint4 *>(gp) = buf.u;
            }
        }
    } else {
        for (int idx = threadIdx.x; idx < nt * kPairs; idx += kThreads) {
            const int r = idx / kPairs, pr = idx % kPairs;
            const int seg = r / L, j = r % L;
            const int c = c0 + 2 * pr;
            T *gp = g + (row0 + r) * C + c;
            W &word = sw[(pr * kSegs + seg) * (L + 1) + j];
            if (TO_SMEM) {
                float2 f;
                f.x = c < C ? Elem<T>::get(gp) : 0.f;
                f.y = c + 1 < C ? Elem<T>::get(gp + 1) : 0.f;
                word = Word<T>::from_f2(f);
            } else {
                float2 f = Word<T>::to_f2(word);
                if (c < C) Elem<T>::put(gp, f.x);
                if (c + 1 < C) Elem<T>::put(gp + 1, f.y);
            }
        }
    }
}

template <typename T, int L>
__global__ void __launch_bounds__(kThreads)
wkv4_scan_kernel(int64_t B, int64_t T_len, int64_t C, const float *__restrict__ w,
                 const float *__restrict__ u, const T *__restrict__ k, const T *__restrict__ v,
                 const float *s0, T *__restrict__ y, float *sT)
{
    using W = typename Word<T>::type;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    W *sk = reinterpret_cast<W *>(smem_raw);
    W *sv = sk + kPairs * kSegs * (L + 1);

    const int64_t cblocks = (C + kCh - 1) / kCh;
    const int64_t b = blockIdx.x / cblocks;
    const int c0 = static_cast<int>((blockIdx.x % cblocks) * kCh);
    const int pr = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ca = c0 + 2 * pr, cb = ca + 1;
    const bool va = ca < C, vb = cb < C;
    const bool vec = (c0 + kCh <= C) && (C % 8 == 0);

    const float w2a = va ? w[ca] * kLog2e : 0.f, w2b = vb ? w[cb] * kLog2e : 0.f;
    const float u2a = va ? u[ca] * kLog2e : 0.f, u2b = vb ? u[cb] * kLog2e : 0.f;

    const St empty{0.f, 0.f, kPEmpty};
    St carry_a = empty, carry_b = empty;
    if (s0) {
        const float *sp = s0 + b * 3 * C;
        if (va && sp[C + ca] != 0.f)
            carry_a = {sp[ca], sp[C + ca], fmaxf(sp[2 * C + ca] * kLog2e, kPEmpty)};
        if (vb && sp[C + cb] != 0.f)
            carry_b = {sp[cb], sp[C + cb], fmaxf(sp[2 * C + cb] * kLog2e, kPEmpty)};
    }

    const T *kb = k + b * T_len * C;
    const T *vbp = v + b * T_len * C;
    T *yb = y + b * T_len * C;
    const W *mk = sk + (pr * kSegs + lane) * (L + 1);
    const W *mv = sv + (pr * kSegs + lane) * (L + 1);
    W *my = sk + (pr * kSegs + lane) * (L + 1);

    for (int64_t t0 = 0; t0 < T_len; t0 += kSegs * L) {
        const int64_t rem = T_len - t0;
        const int nt = rem < kSegs * L ? static_cast<int>(rem) : kSegs * L;
        move_tile<T, L, true>(sk, const_cast<T *>(kb), t0, nt, C, c0, vec);
        move_tile<T, L, true>(sv, const_cast<T *>(vbp), t0, nt, C, c0, vec);
        __syncthreads();

        // pass 1: local summary of this lane's segment
        const int nv = max(0, min(L, nt - lane * L));
        St la = empty, lb = empty;
        for (int j = 0; j < nv; ++j) {
            const float2 kk = Word<T>::to_f2(mk[j]);
            const float2 vv = Word<T>::to_f2(mv[j]);
            update(la, kk.x * kLog2e, vv.x, w2a);
            update(lb, kk.y * kLog2e, vv.y, w2b);
        }

        // inclusive scan over lanes (segment order) with segment lengths
        float n_inc = static_cast<float>(nv);
#pragma unroll
        for (int off = 1; off < kSegs; off <<= 1) {
            const St oa = shfl_up(la, off), ob = shfl_up(lb, off);
            const float on = __shfl_up_sync(0xffffffffu, n_inc, off);
            if (lane >= off) {
                la = combine(oa, la, n_inc * w2a);
                lb = combine(ob, lb, n_inc * w2b);
                n_inc += on;
            }
        }
        // exclusive prefix, then fold in the carry from earlier tiles
        St ea = shfl_up(la, 1), eb = shfl_up(lb, 1);
        float n_exc = __shfl_up_sync(0xffffffffu, n_inc, 1);
        if (lane == 0) {
            ea = empty;
            eb = empty;
            n_exc = 0.f;
        }
        St pa = combine(carry_a, ea, n_exc * w2a);
        St pb = combine(carry_b, eb, n_exc * w2b);
        const St ta = shfl_idx(la, kSegs - 1), tb = shfl_idx(lb, kSegs - 1);
        const float n_tot = __shfl_sync(0xffffffffu, n_inc, kSegs - 1);
        carry_a = combine(carry_a, ta, n_tot * w2a);
        carry_b = combine(carry_b, tb, n_tot * w2b);

        // pass 2: outputs from the exact incoming state; y replaces k in place
        for (int j = 0; j < nv; ++j) {
            const float2 kk = Word<T>::to_f2(mk[j]);
            const float2 vv = Word<T>::to_f2(mv[j]);
            const float k2a = kk.x * kLog2e, k2b = kk.y * kLog2e;
            float2 o;
            o.x = output(pa, k2a, vv.x, u2a);
            o.y = output(pb, k2b, vv.y, u2b);
            update(pa, k2a, vv.x, w2a);
            update(pb, k2b, vv.y, w2b);
            my[j] = Word<T>::from_f2(o);
        }
        __syncthreads();
        move_tile<T, L, false>(sk, yb, t0, nt, C, c0, vec);
        __syncthreads();
    }

    if (sT && lane == 0) {
        float *sp = sT + b * 3 * C;
        if (va) {
            const bool e = carry_a.b == 0.f;
            sp[ca] = carry_a.a;
            sp[C + ca] = carry_a.b;
            sp[2 * C + ca] = e ? kPEmpty : carry_a.p * kLn2;
        }
        if (vb) {
            const bool e = carry_b.b == 0.f;
            sp[cb] = carry_b.a;
            sp[C + cb] = carry_b.b;
            sp[2 * C + cb] = e ? kPEmpty : carry_b.p * kLn2;
        }
    }
}

template <typename T, int L>
cudaError_t launch_L(const Wkv4Args &a, cudaStream_t s)
{
    using W = typename Word<T>::type;
    const size_t smem = 2ull * kPairs * kSegs * (L + 1) * sizeof(W);
    auto kern = wkv4_scan_kernel<T, L>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int64_t blocks = a.B * ((a.C + kCh - 1) / kCh);
    if (blocks == 0) return cudaSuccess;
    kern<<<static_cast<unsigned>(blocks), kThreads, smem, s>>>(
        a.B, a.T, a.C, a.w, a.u, static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.s0,
        static_cast<T *>(a.y), a.sT);
    return cudaGetLastError();
}

template <typename T, int LMAX>
cudaError_t launch_T(const Wkv4Args &a, cudaStream_t s)
{
    const int64_t per_seg = (a.T + kSegs - 1) / kSegs;
    if (per_seg <= 1) return launch_L<T, 1>(a, s);
    if (per_seg <= 2) return launch_L<T, 2>(a, s);
    if (per_seg <= 4) return launch_L<T, 4>(a, s);
    if (per_seg <= 8) return launch_L<T, 8>(a, s);
    if (LMAX == 16 || per_seg <= 16) return launch_L<T, 16>(a, s);
    return launch_L<T, LMAX>(a, s);
}

}  // namespace

cudaError_t wkv4_launch(const Wkv4Args &a, cudaStream_t s)
{
    if (a.B * ((a.C + kCh - 1) / kCh) > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    return a.bf16 ? launch_T<__nv_bfloat16, 32>(a, s) : launch_T<float, 16>(a, s);
}

}  // namespace wkv
