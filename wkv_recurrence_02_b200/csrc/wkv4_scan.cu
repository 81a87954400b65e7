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
//           segment's largest and smallest key are noted on the way, and the summary is
//           renormalised (the denominator's binary exponent moved into the reference) so
//           that the scan compares states by their true magnitude.  (The TMA kernel's
//           bf16 path instead takes the segment's largest exponent, less 15, as reference
//           and keeps every weight as fp16 in its k slot for pass 2; see that kernel.);
//   scan    a 5-step warp shuffle scan combines segment summaries across lanes, and the
//           carry from earlier tiles (or s0) is folded in;
//   pass 2  each lane re-walks its segment from its exact incoming state.  When every
//           term lies within 2^60 of the segment's largest exponent (the normal case)
//           the walk uses that fixed reference: one ex2 per key weight (none where pass
//           1's stored weight is read back) and one reciprocal per output; otherwise it
//           repeats the running-maximum step, which is exact for any inputs.
// Both channels of a lane are carried in 64-bit register pairs and advanced with packed
// f32x2 arithmetic.
//
// Two kernels share this scan; both use one CTA per batch row x 16 channels and
// lane = segment:
//   wkv4_tma_kernel (the default, used when the row pitch is a multiple of 16 bytes, the
//     segment length L divides T and T/L >= 32): the k and v tiles arrive by TMA as
//     token-index-major blocks (block i = token i of all 32 segments); each warp holds one
//     8-byte half of a 16-byte unit of channels; warp 0 issues the first tile's copies
//     before the CTA reads its parameters; pass 2 writes each lane's y rows straight to
//     global memory as it produces them.
//   wkv4_scan_kernel (every other shape: odd C, unaligned pointers, L not dividing T):
//     warp = channel pair (2 channels per lane); k and v tiles are copied with cp.async
//     into a [pair][segment][L+1] layout (the +1 pad and a 4-word skew per pair make both
//     the row-contiguous fill and the lane-strided reads conflict-free); y overwrites k's
//     words in place and is written back with row-contiguous stores.
#include "wkv_internal.cuh"

#include <mutex>

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
// Both reciprocals from one: 1/x = y / (x y) and 1/y = x / (x y).  For 2^-60 <= x, y <= 2^60
// the product stays a normal float; the result carries two more roundings than rcp2.
__device__ __forceinline__ P2 rcp2_shared(P2 x)
{
    const float r = rcp(lo(x) * hi(x));
    return mul2(pk(hi(x), lo(x)), pk(r, r));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

struct St {
    float a, b, p;
};

// (a, b, p) with b's binary exponent moved into p, so that 1 <= b < 4.  A summary taken
// against a reference below its largest term can have b up to 2^127; combining it with a
// later state by the larger exponent p would then flush its (still significant) weight to
// zero, so pass-1 summaries are brought to this form first.  Requires b >= 1.
__device__ __forceinline__ St normalized(float a, float b, float p)
{
    int e = ((__float_as_int(b) >> 23) & 0xff) - 127;
    e = e < 126 ? e : 126;
    const float s = __int_as_float((127 - e) << 23);  // 2^-e, exact
    return {a * s, b * s, p + static_cast<float>(e)};
}

// State `e` (earlier), followed by a block whose local state is `l` and whose total
// log2-decay is nw (= its length times w in log2 units).
__device__ __forceinline__ St combine(St e, St l, float nw)
{
    const float pe = e.p - nw;
    const float d = pe - l.p;
    const float x = ex2(-fabsf(d));  // the smaller side's factor; the larger side's is 1
    const bool early = d >= 0.f;
    const float fe = early ? 1.f : x, fl = early ? x : 1.f;
    return {fmaf(e.a, fe, l.a * fl), fmaf(e.b, fe, l.b * fl), early ? pe : l.p};
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
                 const float *s0, T *__restrict__ y, float *sT, int *status)
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
    if (kDebugBounds) {  // the batch row, this lane's shared-memory segment, the state entries
        const bool ok = in_bounds(status, b, 1, B) && in_bounds(status, widx<L>(pr, lane, 0), L + 1, tile_words<L>()) &&
                        in_bounds(status, b * 3 * C + 2 * C + (va ? ca : 0), 1, B * 3 * C);
        if (!__syncthreads_and(ok)) return;
    }

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
        // debug build: the tile's rows of k, v and y lie inside [B, T, C]
        if (kDebugBounds && !__syncthreads_and(in_bounds(status, (b * T_len + t0) * C, nt * C, B * T_len * C)))
            break;
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
            // the sums must be finite (a weight above 2^127, or a product with v, overflows)
            if (w2a >= 0.f && w2b >= 0.f && Ba <= 3.0e38f && Bb <= 3.0e38f && fabsf(lo(A)) <= 3.0e38f &&
                fabsf(hi(A)) <= 3.0e38f) {
                la = normalized(lo(A), Ba, -lo(nF));
                lb = normalized(hi(A), Bb, -hi(nF));
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

// ===================================================================== TMA-fed variant
// Used when a 16-channel block of k, v, y can be addressed by the tensor-memory
// accelerator (row pitch C * element size a multiple of 16 bytes, 16-byte aligned bases).
// Same algorithm and segment structure as above, different data movement:
//   * one CTA = one batch row x 16 channels; warp h = one 8-byte half of a 16-byte unit
//     of channels (4 bf16 or 2 fp32, carried as f32x2 pairs: 4 or 8 warps), lane = segment;
//   * the tile is held token-index-major: block i (128-byte aligned, as tensor copies
//     require) holds row i of all 32 segments, 16 channels each, and arrives as one TMA
//     box over a 4-D view (channel, i, segment, batch) of [B, T, C] -- exact when L
//     divides T, which the launcher requires;
//   * y replaces k in place and leaves as one TMA store per block (clipped at the last
//     segment and at C);
//   * two tile buffers: tile tau+1 is loaded while tile tau is scanned, and tile tau's
//     store drains while tile tau+1 is scanned.

// Scalar access to the channels of a lane (the exact fallback paths) and the tensor-map
// element type.
template <typename T> struct Unit;
template <> struct Unit<__nv_bfloat16> {
    __device__ static float get(const unsigned char *unit, int n)
    {
        return __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(unit)[n]);
    }
    __device__ static void put(unsigned char *unit, int n, float x)
    {
        reinterpret_cast<__nv_bfloat16 *>(unit)[n] = __float2bfloat16_rn(x);
    }
    static constexpr CUtensorMapDataType kMapType = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};
template <> struct Unit<float> {
    __device__ static float get(const unsigned char *unit, int n) { return reinterpret_cast<const float *>(unit)[n]; }
    __device__ static void put(unsigned char *unit, int n, float x) { reinterpret_cast<float *>(unit)[n] = x; }
    static constexpr CUtensorMapDataType kMapType = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
};

// The channels one lane owns in a token row: one 8-byte half of a 16-byte unit (4 bf16 or 2
// fp32 channels).  Two warps share each unit, so a CTA of 16 channels runs 4 (bf16) or 8
// (fp32) warps and each lane carries half the registers of a whole-unit lane.
template <typename T> struct Lane;
template <> struct Lane<__nv_bfloat16> {
    static constexpr int NC = 4;
    __device__ static uint2 load(const unsigned char *p) { return *reinterpret_cast<const uint2 *>(p); }
    __device__ static void store(unsigned char *p, uint2 x) { *reinterpret_cast<uint2 *>(p) = x; }
    __device__ static void unpack(uint2 u, P2 (&x)[2])
    {
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int q = 0; q < 2; ++q)
            asm("mov.b64 %0, {%1, %2};" : "=l"(x[q].r) : "r"(w[q] << 16), "r"(w[q] & 0xFFFF0000u));
    }
    __device__ static uint2 pack(const P2 (&x)[2])
    {
        uint32_t w[2];
#pragma unroll
        for (int q = 0; q < 2; ++q)
            asm("{\n\t.reg .f32 l, h;\n\tmov.b64 {l, h}, %1;\n\tcvt.rn.bf16x2.f32 %0, h, l;\n\t}"
                : "=r"(w[q])
                : "l"(x[q].r));
        return make_uint2(w[0], w[1]);
    }
};
template <> struct Lane<float> {
    static constexpr int NC = 2;
    __device__ static uint2 load(const unsigned char *p) { return *reinterpret_cast<const uint2 *>(p); }
    __device__ static void store(unsigned char *p, uint2 x) { *reinterpret_cast<uint2 *>(p) = x; }
    __device__ static void unpack(uint2 u, P2 (&x)[1]) { x[0] = pk(__uint_as_float(u.x), __uint_as_float(u.y)); }
    __device__ static uint2 pack(const P2 (&x)[1]) { return make_uint2(__float_as_uint(lo(x[0])), __float_as_uint(hi(x[0]))); }
};

// running min / max of a lane's keys
template <typename T> struct LaneRange;
template <> struct LaneRange<__nv_bfloat16> {
    __nv_bfloat162 mx[2], mn[2];
    __device__ void init()
    {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            mx[q] = __floats2bfloat162_rn(-3.0e38f, -3.0e38f);
            mn[q] = __floats2bfloat162_rn(3.0e38f, 3.0e38f);
        }
    }
    __device__ void add(uint2 u)
    {
        const uint32_t w[2] = {u.x, u.y};
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162 *>(&w[q]);
            mx[q] = __hmax2(mx[q], x);
            mn[q] = __hmin2(mn[q], x);
        }
    }
    __device__ float max(int n) const { return n & 1 ? __high2float(mx[n >> 1]) : __low2float(mx[n >> 1]); }
    __device__ float min(int n) const { return n & 1 ? __high2float(mn[n >> 1]) : __low2float(mn[n >> 1]); }
};
template <> struct LaneRange<float> {
    float mx[2], mn[2];
    __device__ void init()
    {
        mx[0] = mx[1] = -3.4e38f;
        mn[0] = mn[1] = 3.4e38f;
    }
    __device__ void add(uint2 u)
    {
        const float x[2] = {__uint_as_float(u.x), __uint_as_float(u.y)};
#pragma unroll
        for (int n = 0; n < 2; ++n) {
            mx[n] = fmaxf(mx[n], x[n]);
            mn[n] = fminf(mn[n], x[n]);
        }
    }
    __device__ float max(int n) const { return mx[n]; }
    __device__ float min(int n) const { return mn[n]; }
};

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred P;\n\tmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, P;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(phase)
                 : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t phase, uint32_t limit)
{
    for (uint32_t it = 0; it < limit; ++it)
        if (mbar_try(bar, phase)) return true;
    return false;
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2,
                                            int c3, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
                 : "memory");
}
struct TmaParams {
    int64_t T, C, B;
    const float *w, *u, *s0;
    float *sT;
    void *y;  // [B, T, C] of the kernel's element type
    int *status;
    uint32_t spin_limit;
    const void *k;  // [B, T, C]: the exact paths' keys once the tile's slots hold weights
};

// Four fp32 weights as fp16 in a lane's 8-byte k slot, and back.
template <int N>
__device__ __forceinline__ uint2 pack_h4(const P2 (&e)[N])
{
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int q = 0; q < N; ++q)
        asm("{\n\t.reg .f32 l, h;\n\tmov.b64 {l, h}, %1;\n\tcvt.rn.f16x2.f32 %0, h, l;\n\t}" : "=r"(w[q]) : "l"(e[q].r));
    return make_uint2(w[0], w[1]);
}
template <int N>
__device__ __forceinline__ void unpack_h4(uint2 u, P2 (&e)[N])
{
    const uint32_t w[2] = {u.x, u.y};
#pragma unroll
    for (int q = 0; q < N; ++q)
        asm("{\n\t.reg .f16 a, b;\n\t.reg .f32 l, h;\n\tmov.b32 {a, b}, %1;\n\tcvt.f32.f16 l, a;\n\t"
            "cvt.f32.f16 h, b;\n\tmov.b64 %0, {l, h};\n\t}"
            : "=l"(e[q].r)
            : "r"(w[q]));
}
constexpr float kHalfShift = 15.f;  // stored weights are 2^{k - Rf} with Rf 15 below the largest exponent
constexpr float kHalfSpan = 13.f;   // ... and stay fp16 normals (>= 2^-14) while k - Rf >= -13

template <typename T, int L, int NB>
__global__ void __launch_bounds__(32 * (kCh / Lane<T>::NC), 3)
wkv4_tma_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                const TmaParams p)
{
    constexpr int NC = Lane<T>::NC;              // channels per lane
    constexpr int NP = NC / 2;                   // f32x2 pairs per lane
    constexpr int RB = kCh * sizeof(T);          // bytes of one token row (16 channels)
    constexpr int BLK = kSegs * RB;              // bytes of block i: row i of every segment
    // NB buffers (tile tau in buffer tau % NB), each k blocks then v blocks; NB mbarriers.
    // With one buffer the launcher guarantees a single tile.
    extern __shared__ unsigned char smem_raw[];
    // aligned by an offset on the __shared__ array itself (not through an integer), so the
    // compiler keeps the shared state space: its accesses are shared loads and stores, which it
    // may reorder freely around global ones
    unsigned char *sbase = smem_raw + ((128u - (smem_u32(smem_raw) & 127u)) & 127u);
    const uint32_t bar0 = smem_u32(sbase + NB * 2 * L * BLK);  // + 8 * buffer
    // [warp][unit][(a, b, p) x NC channels, segment count]: each warp's scan total
    float *wtot = reinterpret_cast<float *>(sbase + NB * 2 * L * BLK + 8 * NB);

    const int64_t C = p.C, T_len = p.T;
    const int64_t cblocks = (C + kCh - 1) / kCh;
    const int b = static_cast<int>(blockIdx.x / cblocks);
    const int c0 = static_cast<int>((blockIdx.x % cblocks) * kCh);
    // Lanes: a row of block i (token i of all 32 segments, 16 channels each) is 32 x RB bytes;
    // thread x reads its 8 bytes at 8 x, so each warp reads 256 contiguous bytes (no bank
    // conflicts).  That makes lane l of warp h the unit q = l % U (NC channels) of segment
    // h * SPW + l / U, with U units per row and SPW segments per warp.
    constexpr int U = kCh / NC, SPW = kSegs / U;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q = lane % U, seg_l = h * SPW + lane / U;  // this lane's unit and segment
    const int cb = c0 + NC * q;                          // first channel of this lane
    if (kDebugBounds) {  // the batch row; this lane's state entries; its units inside a buffer
        const bool ok = in_bounds(p.status, b, 1, p.B) &&
                        in_bounds(p.status, 8 * static_cast<int>(threadIdx.x) + (L - 1) * BLK,
                                  NC * static_cast<int>(sizeof(T)), L * BLK) &&
                        (cb >= C || in_bounds(p.status, static_cast<int64_t>(b) * 3 * C + 2 * C + cb, 1, p.B * 3 * C));
        if (!__syncthreads_and(ok)) return;
    }
    const int nsegs = static_cast<int>(T_len / L);  // L divides T
    const int ntiles = (nsegs + kSegs - 1) / kSegs;
    // warp 0: lane i brings block i of k and v of tile tl into its buffer
    auto issue = [&](int tl) {
        unsigned char *bk = sbase + (tl % NB) * 2 * L * BLK;
        const uint32_t bar = bar0 + 8 * (tl % NB);
        if (lane == 0) mbar_expect_tx(bar, 2u * L * BLK);
        __syncwarp();
        // debug build: channel block on a 16-byte boundary inside C, the tile's first segment
        // inside T / L (a copy that fails is not issued; its wait then runs out)
        if (lane < L && tma_coord_ok(p.status, c0, static_cast<int>(sizeof(T)), C, static_cast<int64_t>(kSegs) * tl,
                                     T_len / L)) {
            tma_load_4d(smem_u32(bk + lane * BLK), &map_k, c0, lane, kSegs * tl, b, bar);
            tma_load_4d(smem_u32(bk + L * BLK + lane * BLK), &map_v, c0, lane, kSegs * tl, b, bar);
        }
    };
    // the first tile's copies leave before anything else: the parameter loads below then
    // overlap them instead of delaying them
    if (h == 0) {
        if (lane == 0) {
            for (int i = 0; i < NB; ++i) mbar_init(bar0 + 8 * i, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncwarp();
        if (ntiles > 0) issue(0);
    }

    const St empty{0.f, 0.f, kPEmpty};
    float w2[NC], u2[NC];
    P2 dd[NP], ub[NP];
    St carry[NC];
#pragma unroll
    for (int n = 0; n < NC; ++n) {
        const int c = cb + n;
        const bool ok = c < C;
        w2[n] = ok ? p.w[c] * kLog2e : 0.f;
        u2[n] = ok ? p.u[c] * kLog2e : 0.f;
        carry[n] = empty;
        if (p.s0 && ok) {
            const float *sp = p.s0 + static_cast<int64_t>(b) * 3 * C;
            if (sp[C + c] != 0.f) carry[n] = {sp[c], sp[C + c], fmaxf(sp[2 * C + c] * kLog2e, kPEmpty)};
        }
    }
#pragma unroll
    for (int q = 0; q < NP; ++q) {
        dd[q] = pk(ex2(-w2[2 * q]), ex2(-w2[2 * q + 1]));  // per-step decay factors
        ub[q] = pk(ex2(u2[2 * q]), ex2(u2[2 * q + 1]));    // bonus factors
    }
    const P2 l2e = pk(kLog2e, kLog2e), nl2e = pk(-kLog2e, -kLog2e);
    __syncthreads();
    int abort = 0, tile = 0, issued = ntiles > 0 ? 1 : 0;
    for (; tile < ntiles; ++tile) {
        const int seg0 = kSegs * tile;
        if (NB > 1 && tile + 1 < ntiles && h == 0) {
            // the next tile goes to the other buffer, which every thread has finished reading
            // (the barrier at the end of the previous tile)
            issue(tile + 1);
            ++issued;
        }
        unsigned char *sk = sbase + (tile % NB) * 2 * L * BLK;
        const unsigned char *sv = sk + L * BLK;
        abort = __syncthreads_or(!mbar_wait(bar0 + 8 * (tile % NB), (tile / NB) & 1, p.spin_limit));
        if (abort) break;
        // this lane's unit in row 0 of its segment; row i is BLK bytes further
        unsigned char *uk = sk + 8 * threadIdx.x;
        const unsigned char *uv = sv + 8 * threadIdx.x;
        const int nv = seg0 + seg_l < nsegs ? L : 0;

        // pass 1: local summaries and the key range.  bf16 tiles take the segment's largest
        // exponent (largest key, plus u when u > 0) less kHalfShift as the reference Rf, so
        // that every weight 2^{k - Rf} lies in [2^-13, 2^15] when the keys' spread allows
        // (f16ok); each weight then goes back into its k slot as fp16 and pass 2 reads it
        // instead of forming it again.  fp32 tiles take the segment's last key.
        St la[NC];
        LaneRange<T> kr;
        kr.init();
#pragma unroll
        for (int n = 0; n < NC; ++n) la[n] = empty;
        constexpr bool kReuse = sizeof(T) == 2;
        bool f16ok = kReuse;
        float Rf[NC] = {};
        // this lane's keys in global memory: the exact paths read them there once the tile's
        // k slots may hold weights
        const int64_t krow = (static_cast<int64_t>(b) * T_len + static_cast<int64_t>(seg0 + seg_l) * L) * C + cb;
        auto key = [&](int i, int n) -> float {  // key n of the segment's row i, exact paths
            if constexpr (kReuse) {
                const int64_t at = krow + static_cast<int64_t>(i) * C + n;
                return cb < C && in_bounds(p.status, at, 1, p.B * T_len * C)
                           ? Elem<T>::get(static_cast<const T *>(p.k) + at)
                           : 0.f;
            } else {
                return Unit<T>::get(uk + i * BLK, n);
            }
        };
        if (nv > 0) {
            P2 nF[NP], A[NP], Bs[NP];
            if constexpr (kReuse) {
#pragma unroll
                for (int i = 0; i < L; ++i)
                    if (i < nv) kr.add(Lane<T>::load(uk + i * BLK));
#pragma unroll
                for (int n = 0; n < NC; ++n) {
                    Rf[n] = kr.max(n) * kLog2e + fmaxf(u2[n], 0.f) - kHalfShift;
                    f16ok = f16ok && Rf[n] - kr.min(n) * kLog2e <= kHalfSpan;
                }
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    nF[q] = pk(-Rf[2 * q], -Rf[2 * q + 1]);
                    A[q] = pk(0.f, 0.f);
                    Bs[q] = A[q];
                }
            } else {
                P2 kl[NP];
                Lane<T>::unpack(Lane<T>::load(uk + (nv - 1) * BLK), kl);
#pragma unroll
                for (int q = 0; q < NP; ++q) {
                    nF[q] = mul2(kl[q], nl2e);
                    A[q] = pk(0.f, 0.f);
                    Bs[q] = A[q];
                }
            }
#pragma unroll
            for (int i = 0; i < L; ++i) {
                if (i < nv) {
                    const uint2 ku = Lane<T>::load(uk + i * BLK);
                    const uint2 vu = Lane<T>::load(uv + i * BLK);
                    if constexpr (!kReuse) kr.add(ku);
                    P2 kk[NP], vv[NP], Ek[NP];
                    Lane<T>::unpack(ku, kk);
                    Lane<T>::unpack(vu, vv);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const P2 E = ex2_2(fma2(kk[q], l2e, nF[q]));
                        A[q] = fma2(dd[q], A[q], mul2(E, vv[q]));
                        Bs[q] = fma2(dd[q], Bs[q], E);
                        Ek[q] = E;
                    }
                    if constexpr (kReuse) {
                        if (f16ok) Lane<T>::store(uk + i * BLK, pack_h4(Ek));
                    }
                }
            }
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                const P2 a2 = A[n >> 1], b2 = Bs[n >> 1], f2 = nF[n >> 1];
                const float an = n & 1 ? hi(a2) : lo(a2), bn = n & 1 ? hi(b2) : lo(b2);
                const float fn = n & 1 ? hi(f2) : lo(f2);
                if (w2[n] >= 0.f && bn <= 3.0e38f && fabsf(an) <= 3.0e38f && (!kReuse || bn >= 0x1p-100f)) {
                    la[n] = normalized(an, bn, -fn);
                } else {  // a weight overflowed or underflowed (or negative decay): running-maximum steps
                    St s = empty;
                    for (int i = 0; i < nv; ++i) update(s, key(i, n) * kLog2e, Unit<T>::get(uv + i * BLK, n), w2[n]);
                    la[n] = s;
                }
            }
        }
        // inclusive scan over this warp's segments (lanes U apart share a unit) with segment
        // lengths; the warps' totals then meet in shared memory, and each lane folds the
        // carry from earlier tiles, the earlier warps' totals and its warp's exclusive
        // prefix, in segment order
        float n_inc = static_cast<float>(nv);
#pragma unroll
        for (int off = U; off < 32; off <<= 1) {
            const float on = __shfl_up_sync(0xffffffffu, n_inc, off);
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                const St o = shfl_up(la[n], off);
                if (lane >= off) la[n] = combine(o, la[n], n_inc * w2[n]);
            }
            if (lane >= off) n_inc += on;
        }
        float n_exc = __shfl_up_sync(0xffffffffu, n_inc, U);
        if (lane < U) n_exc = 0.f;
        if (lane >= 32 - U) {  // the warp's total for unit q
            float *tw = wtot + (h * U + q) * (3 * NC + 1);
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                tw[3 * n] = la[n].a;
                tw[3 * n + 1] = la[n].b;
                tw[3 * n + 2] = la[n].p;
            }
            tw[3 * NC] = n_inc;
        }
        __syncthreads();
        // the state entering this lane's segment (carry, earlier warps, earlier lanes); the
        // state after the whole tile only where a later tile or sT needs it
        St pa[NC];
        const bool need_all = tile + 1 < ntiles || p.sT != nullptr;
        St before[NC];
#pragma unroll
        for (int n = 0; n < NC; ++n) before[n] = carry[n];
        for (int hw = 0; hw < h; ++hw) {
            const float *tw = wtot + (hw * U + q) * (3 * NC + 1);
#pragma unroll
            for (int n = 0; n < NC; ++n)
                before[n] = combine(before[n], St{tw[3 * n], tw[3 * n + 1], tw[3 * n + 2]}, tw[3 * NC] * w2[n]);
        }
#pragma unroll
        for (int n = 0; n < NC; ++n) {
            St e = shfl_up(la[n], U);
            if (lane < U) e = empty;
            pa[n] = combine(before[n], e, n_exc * w2[n]);
        }
        if (need_all) {
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                St all = carry[n];
#pragma unroll
                for (int hw = 0; hw < kCh / NC; ++hw) {
                    const float *tw = wtot + (hw * U + q) * (3 * NC + 1);
                    const St t{tw[3 * n], tw[3 * n + 1], tw[3 * n + 2]};
                    all = combine(all, t, tw[3 * NC] * w2[n]);
                }
                carry[n] = all;
            }
        }
        // pass 2: outputs from the exact incoming state; each lane writes its y rows to global
        // memory as it goes (8 bytes per row: with every lane of a warp, 32 contiguous bytes of
        // each of 8 segments), so the stores overlap the scan
        T *yrow = static_cast<T *>(p.y) + (static_cast<int64_t>(b) * T_len + static_cast<int64_t>(seg0 + seg_l) * L) * C + cb;
        const bool ystore = nv > 0 && cb < C &&  // debug build: the segment's rows inside y
                            in_bounds(p.status, (static_cast<int64_t>(b) * T_len + static_cast<int64_t>(seg0 + seg_l) * L) * C + cb,
                                      NC, p.B * T_len * C) &&
                            in_bounds(p.status, (static_cast<int64_t>(b) * T_len + static_cast<int64_t>(seg0 + seg_l) * L + L - 1) * C + cb,
                                      NC, p.B * T_len * C);
        bool fixed = true;
        float F[NC];
#pragma unroll
        for (int n = 0; n < NC; ++n) {
            F[n] = fmaxf(pa[n].p, kr.max(n) * kLog2e + fmaxf(u2[n], 0.f));
            fixed = fixed && w2[n] >= 0.f && fabsf(u2[n]) <= kFrame &&
                    F[n] - (u2[n] + kr.min(n) * kLog2e) <= kFrame;
        }
        if (kReuse && fixed && f16ok) {
            // pass 1's weights 2^{k - Rf}, read back from the k slots and brought to F
            P2 A[NP], Bs[NP], sc[NP], ubs[NP];
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const float s_lo = ex2(pa[2 * q].p - F[2 * q]), s_hi = ex2(pa[2 * q + 1].p - F[2 * q + 1]);
                A[q] = pk(pa[2 * q].a * s_lo, pa[2 * q + 1].a * s_hi);
                Bs[q] = pk(pa[2 * q].b * s_lo, pa[2 * q + 1].b * s_hi);
                sc[q] = pk(ex2(Rf[2 * q] - F[2 * q]), ex2(Rf[2 * q + 1] - F[2 * q + 1]));
                ubs[q] = mul2(ub[q], sc[q]);
            }
#pragma unroll
            for (int i = 0; i < L; ++i) {
                if (i < nv) {
                    const uint2 eu = Lane<T>::load(uk + i * BLK);
                    const uint2 vu = Lane<T>::load(uv + i * BLK);
                    P2 e0[NP], vv[NP], o[NP];
                    unpack_h4(eu, e0);
                    Lane<T>::unpack(vu, vv);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const P2 E = mul2(e0[q], sc[q]);
                        const P2 bE = mul2(ubs[q], e0[q]);
                        o[q] = mul2(fma2(bE, vv[q], A[q]), rcp2_shared(add2(Bs[q], bE)));
                        A[q] = fma2(dd[q], A[q], mul2(E, vv[q]));
                        Bs[q] = fma2(dd[q], Bs[q], E);
                    }
                    if (ystore) *reinterpret_cast<uint2 *>(yrow + static_cast<int64_t>(i) * C) = Lane<T>::pack(o);
                }
            }
        } else if (fixed) {
            // every weight is 2^{x - F} <= 1 and the bonus term keeps the denominator >= 2^-60
            P2 A[NP], Bs[NP], nF[NP];
#pragma unroll
            for (int q = 0; q < NP; ++q) {
                const float s_lo = ex2(pa[2 * q].p - F[2 * q]), s_hi = ex2(pa[2 * q + 1].p - F[2 * q + 1]);
                A[q] = pk(pa[2 * q].a * s_lo, pa[2 * q + 1].a * s_hi);
                Bs[q] = pk(pa[2 * q].b * s_lo, pa[2 * q + 1].b * s_hi);
                nF[q] = pk(-F[2 * q], -F[2 * q + 1]);
            }
#pragma unroll
            for (int i = 0; i < L; ++i) {
                if (i < nv) {
                    const uint2 ku = Lane<T>::load(uk + i * BLK);
                    const uint2 vu = Lane<T>::load(uv + i * BLK);
                    P2 kk[NP], vv[NP], o[NP];
                    Lane<T>::unpack(ku, kk);
                    Lane<T>::unpack(vu, vv);
#pragma unroll
                    for (int q = 0; q < NP; ++q) {
                        const P2 E = ex2_2(fma2(kk[q], l2e, nF[q]));
                        const P2 bE = mul2(ub[q], E);
                        o[q] = mul2(fma2(bE, vv[q], A[q]), rcp2_shared(add2(Bs[q], bE)));
                        A[q] = fma2(dd[q], A[q], mul2(E, vv[q]));
                        Bs[q] = fma2(dd[q], Bs[q], E);
                    }
                    if (ystore) *reinterpret_cast<uint2 *>(yrow + static_cast<int64_t>(i) * C) = Lane<T>::pack(o);
                }
            }
        } else {
            // running-maximum steps, exact for any inputs; channel by channel
#pragma unroll
            for (int n = 0; n < NC; ++n) {
                St s = pa[n];
                for (int i = 0; i < nv; ++i) {
                    const float k2 = key(i, n) * kLog2e, vx = Unit<T>::get(uv + i * BLK, n);
                    const float o = output(s, k2, vx, u2[n]);
                    update(s, k2, vx, w2[n]);
                    if (ystore) Elem<T>::put(yrow + static_cast<int64_t>(i) * C + n, o);
                }
            }
        }
        // every thread is done reading this tile's buffer before it is refilled
        if (kReuse && NB > 1) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncthreads();
    }
    if (abort) {
        record_status(p.status, kStatusTimeout);
        if (threadIdx.x == 0)  // bounded: let the copies in flight land before the CTA exits
            for (int t = tile; t < issued; ++t) mbar_wait(bar0 + 8 * (t % NB), (t / NB) & 1, p.spin_limit);
        __syncthreads();
        return;
    }

    if (p.sT && h == 0 && lane < U) {  // every lane of a unit holds the same carry
        float *sp = p.sT + static_cast<int64_t>(b) * 3 * C;
#pragma unroll
        for (int n = 0; n < NC; ++n) {
            const int c = cb + n;
            if (c < C) {
                const bool e = carry[n].b == 0.f;
                sp[c] = carry[n].a;
                sp[C + c] = carry[n].b;
                sp[2 * C + c] = e ? kPEmpty : carry[n].p * kLn2;
            }
        }
    }
}

template <typename T, int L, int NB>
cudaError_t launch_tma_L(const Wkv4Args &a, cudaStream_t s)
{
    constexpr int NC = Lane<T>::NC;
    constexpr int RB = kCh * sizeof(T);
    constexpr int BLK = kSegs * RB;
    constexpr int kThr = 32 * (kCh / NC);
    constexpr int U = kCh / NC;
    // buffers of k and v blocks, alignment slack, mbarriers, the warps' scan totals
    const size_t smem = NB * 2ull * L * BLK + 128 + 8 * NB + sizeof(float) * (kCh / NC) * U * (3 * NC + 1);
    auto enc = tensor_map_encoder();
    if (!enc) return cudaErrorNotSupported;
    // 4-D view (channel, token within segment, segment, batch row) of [B, T, C]; L divides T
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(a.C), static_cast<cuuint64_t>(L),
                                static_cast<cuuint64_t>(a.T / L), static_cast<cuuint64_t>(a.B)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(a.C * sizeof(T)),
                                   static_cast<cuuint64_t>(L * a.C * sizeof(T)),
                                   static_cast<cuuint64_t>(a.T * a.C * sizeof(T))};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(kCh), 1, static_cast<cuuint32_t>(kSegs), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUtensorMap mk, mv;
    const void *ptrs[2] = {a.k, a.v};
    CUtensorMap *maps[2] = {&mk, &mv};
    for (int i = 0; i < 2; ++i)
        if (enc(maps[i], Unit<T>::kMapType, 4, const_cast<void *>(ptrs[i]), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    auto kern = wkv4_tma_kernel<T, L, NB>;
    {
        // shared-memory attributes, once per device and instantiation
        static std::mutex mu;
        static bool done[64] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
        std::lock_guard<std::mutex> lock(mu);
        if (!done[dev]) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
            if (e != cudaSuccess) return e;
            done[dev] = true;
        }
    }
    const int64_t blocks = a.B * ((a.C + kCh - 1) / kCh);
    const TmaParams prm{a.T, a.C, a.B, a.w, a.u, a.s0, a.sT, a.y, a.status, 1u << 22, a.k};
    kern<<<static_cast<unsigned>(blocks), kThr, smem, s>>>(mk, mv, prm);
    return cudaGetLastError();
}

// Segment length: the smallest power of two giving 32 segments that cover T, capped at LMAX.
int pick_L(int64_t T, int LMAX)
{
    const int64_t per_seg = (T + kSegs - 1) / kSegs;
    int L = 1;
    while (L < per_seg && L < LMAX) L *= 2;
    return L;
}

// One tile (T <= 32 L): one buffer of up to 64 KB.  Several tiles: two buffers of up to
// 32 KB each (half the segment length), so tile tau+1 loads while tile tau is scanned.
// Both keep three CTAs per SM.
template <typename T>
cudaError_t launch_tma_T(const Wkv4Args &a, int L, int NB, cudaStream_t s)
{
    if (NB == 1) {
        switch (L) {
        case 1: return launch_tma_L<T, 1, 1>(a, s);
        case 2: return launch_tma_L<T, 2, 1>(a, s);
        case 4: return launch_tma_L<T, 4, 1>(a, s);
        case 8: return launch_tma_L<T, 8, 1>(a, s);
        case 16: return launch_tma_L<T, 16, 1>(a, s);
        default: break;
        }
        if constexpr (sizeof(T) == 2)
            if (L == 32) return launch_tma_L<T, 32, 1>(a, s);
        return cudaErrorInvalidValue;
    }
    if constexpr (sizeof(T) == 2)
        if (L == 16) return launch_tma_L<T, 16, 2>(a, s);
    if constexpr (sizeof(T) == 4)
        if (L == 8) return launch_tma_L<T, 8, 2>(a, s);
    return cudaErrorInvalidValue;
}

// True when TMA can address the 16-channel blocks: row pitch a multiple of 16 bytes,
// 16-byte aligned bases, coordinates within int32.
bool tma_usable(const Wkv4Args &a)
{
    const int64_t es = a.bf16 ? 2 : 4;
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    return a.T > 0 && a.B > 0 && a.C > 0 && (a.C * es) % 16 == 0 && al16(a.k) && al16(a.v) && al16(a.y) &&
           a.T < (int64_t(1) << 31) - 64 && a.B < (int64_t(1) << 31) && a.C < (int64_t(1) << 31) &&
           tensor_map_encoder() != nullptr;
}

// ======================================================================= decode (T = 1)
// One token per call (serving): one thread per (batch row, NV adjacent channels) applies the
// output and running-maximum update steps above to each (a, b, p) state, which may be
// updated in place (sT == s0).  Grid: x over channel groups, y over batch rows (a loop
// covers rows beyond 65535); loads and stores are coalesced along the channel.
template <typename T, int NV>
__global__ void __launch_bounds__(256)
wkv4_decode_kernel(int64_t B, int64_t C, const float *__restrict__ w, const float *__restrict__ u,
                   const T *__restrict__ k, const T *__restrict__ v, const float *s0, T *__restrict__ y, float *sT,
                   int *status)
{
    const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * NV;
    if (c0 >= C) return;
    if (!in_bounds(status, c0, NV, C)) return;  // debug build: this thread's channels inside C
    float w2[NV], u2[NV];
#pragma unroll
    for (int j = 0; j < NV; ++j) {
        w2[j] = w[c0 + j] * kLog2e;
        u2[j] = u[c0 + j] * kLog2e;
    }
    for (int64_t b = blockIdx.y; b < B; b += gridDim.y) {
        const int64_t i = b * C + c0;
        const float *sp = s0 ? s0 + b * 3 * C : nullptr;
        float *tp = sT ? sT + b * 3 * C : nullptr;
#pragma unroll
        for (int j = 0; j < NV; ++j) {
            const float k2 = Elem<T>::get(k + i + j) * kLog2e, vx = Elem<T>::get(v + i + j);
            St st{0.f, 0.f, kPEmpty};
            if (sp) {
                const float sb = sp[C + c0 + j];
                if (sb != 0.f) st = {sp[c0 + j], sb, fmaxf(sp[2 * C + c0 + j] * kLog2e, kPEmpty)};
            }
            Elem<T>::put(y + i + j, output(st, k2, vx, u2[j]));
            update(st, k2, vx, w2[j]);
            if (tp) {
                tp[c0 + j] = st.a;
                tp[C + c0 + j] = st.b;
                tp[2 * C + c0 + j] = st.b == 0.f ? kPEmpty : st.p * kLn2;
            }
        }
    }
}

// Four adjacent channels of one token row: k, v loads and the y store in one access each.
template <typename T> struct Row4;
template <> struct Row4<float> {
    __device__ static void load(const float *p, float (&x)[4])
    {
        const float4 q = *reinterpret_cast<const float4 *>(p);
        x[0] = q.x, x[1] = q.y, x[2] = q.z, x[3] = q.w;
    }
    __device__ static void store(float *p, const float (&x)[4])
    {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};
template <> struct Row4<__nv_bfloat16> {
    __device__ static void load(const __nv_bfloat16 *p, float (&x)[4])
    {
        const uint2 q = *reinterpret_cast<const uint2 *>(p);
        x[0] = __uint_as_float(q.x << 16), x[1] = __uint_as_float(q.x & 0xFFFF0000u);
        x[2] = __uint_as_float(q.y << 16), x[3] = __uint_as_float(q.y & 0xFFFF0000u);
    }
    __device__ static void store(__nv_bfloat16 *p, const float (&x)[4])
    {
        const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]), hi = __floats2bfloat162_rn(x[2], x[3]);
        *reinterpret_cast<uint2 *>(p) =
            make_uint2(*reinterpret_cast<const uint32_t *>(&lo), *reinterpret_cast<const uint32_t *>(&hi));
    }
};

// The decode step of wkv4_decode_kernel for C a multiple of 4: each thread owns 4 adjacent
// channels, so every state row (a, b, p), w, u, k, v and y moves in one 16- or 8-byte access
// (the launcher's pointers are 16-byte aligned and C % 4 == 0, so every offset is aligned).
template <typename T>
__global__ void __launch_bounds__(256)
wkv4_decode4_kernel(int64_t B, int64_t C, const float *__restrict__ w, const float *__restrict__ u,
                    const T *__restrict__ k, const T *__restrict__ v, const float *s0, T *__restrict__ y, float *sT,
                    int *status)
{
    const int64_t c0 = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
    if (c0 >= C) return;
    if (!in_bounds(status, c0, 4, C)) return;  // debug build: this thread's channels inside C
    const float4 wq = *reinterpret_cast<const float4 *>(w + c0), uq = *reinterpret_cast<const float4 *>(u + c0);
    const float w2[4] = {wq.x * kLog2e, wq.y * kLog2e, wq.z * kLog2e, wq.w * kLog2e};
    const float u2[4] = {uq.x * kLog2e, uq.y * kLog2e, uq.z * kLog2e, uq.w * kLog2e};
    for (int64_t b = blockIdx.y; b < B; b += gridDim.y) {
        const int64_t i = b * C + c0;
        float kk[4], vv[4];
        Row4<T>::load(k + i, kk);
        Row4<T>::load(v + i, vv);
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f}, sq[4] = {0.f, 0.f, 0.f, 0.f};
        if (s0) {
            const float *sp = s0 + b * 3 * C;
            Row4<float>::load(sp + c0, sa);
            Row4<float>::load(sp + C + c0, sb);
            Row4<float>::load(sp + 2 * C + c0, sq);
        }
        float yo[4], na[4], nb[4], np[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float k2 = kk[j] * kLog2e;
            St st{0.f, 0.f, kPEmpty};
            if (sb[j] != 0.f) st = {sa[j], sb[j], fmaxf(sq[j] * kLog2e, kPEmpty)};
            yo[j] = output(st, k2, vv[j], u2[j]);
            update(st, k2, vv[j], w2[j]);
            na[j] = st.a;
            nb[j] = st.b;
            np[j] = st.b == 0.f ? kPEmpty : st.p * kLn2;
        }
        Row4<T>::store(y + i, yo);
        if (sT) {
            float *tp = sT + b * 3 * C;
            Row4<float>::store(tp + c0, na);
            Row4<float>::store(tp + C + c0, nb);
            Row4<float>::store(tp + 2 * C + c0, np);
        }
    }
}

template <typename T, int NV>
cudaError_t launch_decode_v(const Wkv4Args &a, cudaStream_t s)
{
    const int64_t groups = (a.C + NV - 1) / NV;
    const int64_t bx = (groups + 255) / 256;
    if (bx > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    const unsigned by = static_cast<unsigned>(a.B < 65535 ? a.B : 65535);
    if (NV == 4)
        wkv4_decode4_kernel<T><<<dim3(static_cast<unsigned>(bx), by), 256, 0, s>>>(
            a.B, a.C, a.w, a.u, static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.s0,
            static_cast<T *>(a.y), a.sT, a.status);
    else
        wkv4_decode_kernel<T, NV><<<dim3(static_cast<unsigned>(bx), by), 256, 0, s>>>(
            a.B, a.C, a.w, a.u, static_cast<const T *>(a.k), static_cast<const T *>(a.v), a.s0,
            static_cast<T *>(a.y), a.sT, a.status);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_decode(const Wkv4Args &a, cudaStream_t s)
{
    if (a.B == 0 || a.C == 0) return cudaSuccess;
    if (a.C % 4 == 0) return launch_decode_v<T, 4>(a, s);
    return a.C % 2 == 0 ? launch_decode_v<T, 2>(a, s) : launch_decode_v<T, 1>(a, s);
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
        static_cast<T *>(a.y), a.sT, a.status);
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
    if (a.T == 1) return a.bf16 ? launch_decode<__nv_bfloat16>(a, s) : launch_decode<float>(a, s);
    if (a.B * ((a.C + kCh - 1) / kCh) > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (tma_usable(a)) {
        const int lmax = a.bf16 ? 32 : 16;
        int L = pick_L(a.T, lmax), NB = 1;
        if (a.T > static_cast<int64_t>(kSegs) * L) {  // several tiles: two half-size buffers
            L = pick_L(a.T, lmax / 2);
            NB = 2;
        }
        // the 4-D view needs L to divide T; a box spans 32 segments, so T/L >= 32
        if (a.T % L == 0 && a.T / L >= kSegs)
            return a.bf16 ? launch_tma_T<__nv_bfloat16>(a, L, NB, s) : launch_tma_T<float>(a, L, NB, s);
    }
    return a.bf16 ? launch_T<__nv_bfloat16, 32>(a, s) : launch_T<float, 16>(a, s);
}

}  // namespace wkv
