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
// state and its total decay n*w, so T is cut into tiles of 32 segments of L tokens:
//   pass 1  each lane summarises its own segment from the empty state, with the
//           segment's last key as reference: the last token's weight is exactly 1, so
//           the denominator never underflows, and every other weight is a single ex2
//           (the decay a plain multiply).  If a weight overflows (keys more than 2^127
//           apart) the lane redoes its segment with the running-maximum step.  The
//           segment's largest and smallest key are noted on the way;
//   scan    a 5-step warp shuffle scan combines segment summaries across lanes, and the
//           carry from earlier tiles (or s0) is folded in;
//   pass 2  each lane re-walks its segment from its exact incoming state.  When every
//           term lies within 2^60 of the segment's largest exponent (the normal case)
//           the walk uses that fixed reference: one ex2 per key weight and one
//           reciprocal per output; otherwise it repeats the running-maximum step, which
//           is exact for any inputs.
// Both channels of a lane are carried in 64-bit register pairs and advanced with packed
// f32x2 arithmetic.
//
// Layout: one CTA = one batch row x 16 channels; warp = channel pair (2 channels per
// lane), lane = segment.  k and v tiles (32 x L tokens x 16 channels) are copied with
// cp.async straight into a [pair][segment][L+1] layout (the +1 pad and a 4-word skew per
// pair make both the row-contiguous fill and the lane-strided reads conflict-free).
// y overwrites k's words in place and is written back with row-contiguous stores.
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
constexpr float kFrame = 60.f;     // fixed-reference pass 2: allowed spread in log2 units

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 channels in one 64-bit register pair (low half = first channel).
struct P2 {
    unsigned long long r;
};

__device__ __forceinline__ P2 pk(float lo, float hi)
{
    P2 p;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p.r) : "f"(lo), "f"(hi));
    return p;
}
__device__ __forceinline__ float lo(P2 p)
{
    float a;
    asm("{\n\t.reg .f32 t;\n\tmov.b64 {%0, t}, %1;\n\t}" : "=f"(a) : "l"(p.r));
    return a;
}
__device__ __forceinline__ float hi(P2 p)
{
    float b;
    asm("{\n\t.reg .f32 t;\n\tmov.b64 {t, %0}, %1;\n\t}" : "=f"(b) : "l"(p.r));
    return b;
}
__device__ __forceinline__ P2 fma2(P2 a, P2 b, P2 c)
{
    P2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.r) : "l"(a.r), "l"(b.r), "l"(c.r));
    return d;
}
__device__ __forceinline__ P2 mul2(P2 a, P2 b)
{
    P2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}
__device__ __forceinline__ P2 add2(P2 a, P2 b)
{
    P2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}
__device__ __forceinline__ P2 ex2_2(P2 x) { return pk(ex2(lo(x)), ex2(hi(x))); }
__device__ __forceinline__ P2 rcp2(P2 x) { return pk(rcp(lo(x)), rcp(hi(x))); }

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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
    __device__ static P2 unpack(float2 x) { return pk(x.x, x.y); }
    __device__ static float2 to_f2(float2 x) { return x; }
    __device__ static float2 from_f2(float2 x) { return x; }
};
template <> struct Word<__nv_bfloat16> {
    using type = __nv_bfloat162;
    __device__ static P2 unpack(__nv_bfloat162 x)
    {
        const uint32_t w = *reinterpret_cast<uint32_t *>(&x);
        P2 p;
        asm("mov.b64 %0, {%1, %2};" : "=l"(p.r) : "r"(w << 16), "r"(w & 0xFFFF0000u));
        return p;
    }
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

// word index of (pair, segment, j) in one tile buffer
template <int L> __device__ __forceinline__ int widx(int pr, int seg, int j)
{
    return pr * (kSegs * (L + 1) + 4) + seg * (L + 1) + j;
}
template <int L> __host__ __device__ constexpr int tile_words() { return kPairs * (kSegs * (L + 1) + 4); }

// Copies one tile (rows row0 .. row0+nt-1, channels c0..c0+15) of k and v into their
// buffers: thread t always moves pair t % 8 of rows t/8 + 32 i, so every address steps by
// a constant.  Word-granular cp.async when C is even; element loads otherwise.
template <typename T, int L>
__device__ __forceinline__ void fetch_tile(typename Word<T>::type *bk, typename Word<T>::type *bv,
                                           const T *k, const T *v, int64_t row0, int nt, int64_t C, int c0)
{
    using W = typename Word<T>::type;
    constexpr int kRowsPerPass = kThreads / kPairs;  // 32
    const int pr = threadIdx.x % kPairs, r0 = threadIdx.x / kPairs;
    const int c = c0 + 2 * pr;
    const int64_t g0 = (row0 + r0) * C + c;
    const int64_t gstep = kRowsPerPass * C;
    if ((C % 2) == 0 && c + 1 < C) {
        const uint32_t sk = smem_u32(bk), sv = smem_u32(bv);
#pragma unroll 4
        for (int i = 0; i < L; ++i) {
            const int r = r0 + kRowsPerPass * i;
            if (r < nt) {
                const uint32_t off = static_cast<uint32_t>(widx<L>(pr, r / L, r % L) * sizeof(W));
                asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(sk + off), "l"(k + g0 + i * gstep),
                             "n"(sizeof(W)));
                asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(sv + off), "l"(v + g0 + i * gstep),
                             "n"(sizeof(W)));
            }
        }
    } else {
        for (int i = 0; i < L; ++i) {
            const int r = r0 + kRowsPerPass * i;
            if (r < nt) {
                const int64_t g = g0 + i * gstep;
                float2 fk, fv;
                fk.x = c < C ? Elem<T>::get(k + g) : 0.f;
                fk.y = c + 1 < C ? Elem<T>::get(k + g + 1) : 0.f;
                fv.x = c < C ? Elem<T>::get(v + g) : 0.f;
                fv.y = c + 1 < C ? Elem<T>::get(v + g + 1) : 0.f;
                bk[widx<L>(pr, r / L, r % L)] = Word<T>::from_f2(fk);
                bv[widx<L>(pr, r / L, r % L)] = Word<T>::from_f2(fv);
            }
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Writes y (held in the k buffer) of one tile back to global memory.
template <typename T, int L>
__device__ __forceinline__ void store_tile(const typename Word<T>::type *by, T *y, int64_t row0, int nt,
                                           int64_t C, int c0)
{
    using W = typename Word<T>::type;
    constexpr int kWordsPerVec = 16 / sizeof(W);      // 4 (bf16x2) or 2 (float2)
    constexpr int kVecPerRow = kPairs / kWordsPerVec;  // 2 or 4
    if (c0 + kCh <= C && C % 8 == 0) {
        for (int idx = threadIdx.x; idx < nt * kVecPerRow; idx += kThreads) {
            const int r = idx / kVecPerRow, qv = idx % kVecPerRow;
            union {
                uint4 u;
                W w[kWordsPerVec];
            } buf;
#pragma unroll
            for (int m = 0; m < kWordsPerVec; ++m) buf.w[m] = by[widx<L>(qv * kWordsPerVec + m, r / L, r % L)];
            *reinterpret_cast<uint4 *>(y + (row0 + r) * C + c0 + qv * kWordsPerVec * 2) = buf.u;
        }
    } else {
        for (int idx = threadIdx.x; idx < nt * kPairs; idx += kThreads) {
            const int r = idx / kPairs, pr = idx % kPairs;
            const int c = c0 + 2 * pr;
            const float2 f = Word<T>::to_f2(by[widx<L>(pr, r / L, r % L)]);
            T *gp = y + (row0 + r) * C + c;
            if (c < C) Elem<T>::put(gp, f.x);
            if (c + 1 < C) Elem<T>::put(gp + 1, f.y);
        }
    }
}

template <typename T, int L>
__global__ void __launch_bounds__(kThreads, 3)
wkv4_scan_kernel(int64_t B, int64_t T_len, int64_t C, const float *__restrict__ w,
                 const float *__restrict__ u, const T *__restrict__ k, const T *__restrict__ v,
                 const float *s0, T *__restrict__ y, float *sT)
{
    using W = typename Word<T>::type;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    W *bk = reinterpret_cast<W *>(smem_raw);  // [k, v][tile words]
    W *bv = bk + tile_words<L>();
    constexpr int TILE = kSegs * L;

    const int64_t cblocks = (C + kCh - 1) / kCh;
    const int64_t b = blockIdx.x / cblocks;
    const int c0 = static_cast<int>((blockIdx.x % cblocks) * kCh);
    const int pr = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ca = c0 + 2 * pr, cb = ca + 1;
    const bool va = ca < C, vb = cb < C;

    const float w2a = va ? w[ca] * kLog2e : 0.f, w2b = vb ? w[cb] * kLog2e : 0.f;
    const float u2a = va ? u[ca] * kLog2e : 0.f, u2b = vb ? u[cb] * kLog2e : 0.f;
    const P2 dd = pk(ex2(-w2a), ex2(-w2b));   // per-step decay factors
    const P2 ub = pk(ex2(u2a), ex2(u2b));     // bonus factors
    const P2 l2e = pk(kLog2e, kLog2e);

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
    const W *mk = bk + widx<L>(pr, lane, 0);
    const W *mv = bv + widx<L>(pr, lane, 0);
    W *my = bk + widx<L>(pr, lane, 0);

    for (int64_t t0 = 0; t0 < T_len; t0 += TILE) {
        const int64_t rem = T_len - t0;
        const int nt = rem < TILE ? static_cast<int>(rem) : TILE;
        fetch_tile<T, L>(bk, bv, kb, vbp, t0, nt, C, c0);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        const int nv = max(0, min(L, nt - lane * L));

        // pass 1: local summary against the segment's last key; key range
        St la = empty, lb = empty;
        float kmaxa = -3.4e38f, kmaxb = -3.4e38f, kmina = 3.4e38f, kminb = 3.4e38f;
        if (nv > 0) {
            const float2 kl = Word<T>::to_f2(mk[nv - 1]);
            const P2 nF = pk(-kl.x * kLog2e, -kl.y * kLog2e);
            P2 A = pk(0.f, 0.f), Bs = A;
            float kxa = -3.4e38f, kxb = -3.4e38f, kna = 3.4e38f, knb = 3.4e38f;
#pragma unroll 4
            for (int j = 0; j < nv; ++j) {
                const P2 kk = Word<T>::unpack(mk[j]);
                const P2 vv = Word<T>::unpack(mv[j]);
                kxa = fmaxf(kxa, lo(kk));
                kxb = fmaxf(kxb, hi(kk));
                kna = fminf(kna, lo(kk));
                knb = fminf(knb, hi(kk));
                const P2 E = ex2_2(fma2(kk, l2e, nF));
                A = fma2(dd, A, mul2(E, vv));
                Bs = fma2(dd, Bs, E);
            }
            kmaxa = kxa * kLog2e;
            kmaxb = kxb * kLog2e;
            kmina = kna * kLog2e;
            kminb = knb * kLog2e;
            const float Ba = lo(Bs), Bb = hi(Bs);
            if (w2a >= 0.f && w2b >= 0.f && Ba <= 3.0e38f && Bb <= 3.0e38f) {
                la = {lo(A), Ba, -lo(nF)};
                lb = {hi(A), Bb, -hi(nF)};
            } else {
                for (int j = 0; j < nv; ++j) {
                    const float2 kk = Word<T>::to_f2(mk[j]);
                    const float2 vv = Word<T>::to_f2(mv[j]);
                    update(la, kk.x * kLog2e, vv.x, w2a);
                    update(lb, kk.y * kLog2e, vv.y, w2b);
                }
            }
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
        const float Fa = fmaxf(pa.p, kmaxa + fmaxf(u2a, 0.f));
        const float Fb = fmaxf(pb.p, kmaxb + fmaxf(u2b, 0.f));
        const bool fixed = w2a >= 0.f && w2b >= 0.f && fabsf(u2a) <= kFrame && fabsf(u2b) <= kFrame &&
                           Fa - (u2a + kmina) <= kFrame && Fb - (u2b + kminb) <= kFrame;
        if (fixed) {
            // every weight is 2^{x - F} <= 1 and the bonus term keeps the denominator >= 2^-60
            const float sa = ex2(pa.p - Fa), sb = ex2(pb.p - Fb);
            const P2 nF = pk(-Fa, -Fb);
            P2 A = pk(pa.a * sa, pb.a * sb), Bs = pk(pa.b * sa, pb.b * sb);
#pragma unroll 4
            for (int j = 0; j < nv; ++j) {
                const P2 kk = Word<T>::unpack(mk[j]);
                const P2 vv = Word<T>::unpack(mv[j]);
                const P2 E = ex2_2(fma2(kk, l2e, nF));
                const P2 bE = mul2(ub, E);
                const P2 o = mul2(fma2(bE, vv, A), rcp2(add2(Bs, bE)));
                A = fma2(dd, A, mul2(E, vv));
                Bs = fma2(dd, Bs, E);
                my[j] = Word<T>::from_f2(make_float2(lo(o), hi(o)));
            }
        } else {
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
        }
        __syncthreads();
        store_tile<T, L>(bk, yb, t0, nt, C, c0);
        __syncthreads();  // the buffers are refilled by the next tile
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
    const size_t smem = 2ull * tile_words<L>() * sizeof(W);
    auto kern = wkv4_scan_kernel<T, L>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    const int64_t blocks = a.B * ((a.C + kCh - 1) / kCh);
    if (blocks == 0) return cudaSuccess;
    kern<<<static_cast<unsigned>(blocks), kThreads, smem, s>>>(
        a.B, a.T, a.C, a.w, a.u, static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.s0,
        static_cast<T *>(a.y), a.sT);
    return cudaGetLastError();
}

// Segment length: the smallest power of two giving 32 segments that cover T, capped so a
// tile (k and v) keeps 3 CTAs per SM within shared memory.
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
