// wkv6_chunked.cu -- chunked WKV-6 prefill on B200 tensor cores (tcgen05 + TMA + TMEM).
//
// Source: "RWKV-5/6 (Eagle and Finch)", section 4.1.2 (Eagle time mixing: the state is a
// sum of k^T v, each key channel decayed by its w at every step, gain u on the current
// token, receptance applied like a query), section 4.2.2 (Finch: per-token w_t) and
// section 4 (row vectors, matrices act on the right: S[i][j], i = key channel,
// j = value channel).  Per token:  y_t = r_t (S + diag(u) k_t^T v_t),
// S <- diag(w_t) S + k_t^T v_t.  The RWKV-4 paper's parallelisation section motivates
// evaluating the recurrence in time-parallel blocks.
//
// One CTA owns one (batch row, head) and walks its sequence in 64-token chunks.  The
// fp32 state S (64x64) lives in tensor memory for the whole sequence.  Per chunk:
//
//   decay bookkeeping  Each 64-token chunk is 4 sub-blocks of 16.  With P_t the product of
//                      w from the start of t's sub-block through t (running products on
//                      CUDA cores -- no logarithms, no exponentials), every factor used
//                      below is a product of w's and therefore <= 1, except the inverse
//                      1/P_i of the diagonal sub-blocks (guarded, see below).
//   intra-chunk scores A[t][i] = r_t . (k_i * prod_{j=i+1}^{t-1} w_j)  (i < t):
//     off-diagonal     key sub-block b < query sub-block a: reference at the end of b,
//                      Qo_b[t] = r_t * prod_{j=e_b+1}^{t-1} w_j,  Kb[i] = k_i * prod_{j=i+1}^{e_b} w_j,
//                      three tcgen05 MMAs (M=64, N=16, K=64) into TMEM;
//     diagonal         Qd[t] = r_t P_{t-1}, Kd[i] = k_i / P_i, one MMA (N=64), the four
//                      16x16 diagonal blocks used.  If some P in the chunk falls below
//                      2^-60 (very fast decay) the diagonal blocks are instead computed
//                      exactly on CUDA cores from running products of w.
//     A[t][t]          = sum_c r_t[c] u[c] k_t[c]  (the bonus term), on CUDA cores.
//   O  = P V + Qi S_prev        P = causal-masked A in bf16, Qi[t] = r_t * prod_{j<t} w_j
//   S  = diag(D) S_prev + Kh^T V,   Kh[i] = k_i * prod_{j>i} w_j,  D = prod_j w_j
// The five products are tcgen05.mma kind::f16 (bf16 operands from swizzled shared
// memory, fp32 accumulators in TMEM); S_prev is read from TMEM, copied to a bf16
// operand tile and scaled by D in place.  r, k, v, w tiles arrive by TMA (4-D tensor
// maps over [B, T, H, N], 128-byte swizzle, zero fill past T) into a 2-stage ring.
//
// Every mbarrier wait is bounded; on expiry the CTA records RWKV_ERR_TIMEOUT in the
// device status word, waits (bounded) for its own copies and MMAs, frees its tensor
// memory and returns.
#include "wkv_internal.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>

namespace wkv {
namespace {

constexpr int kC = 64;                 // tokens per chunk
constexpr int kN = 64;                 // head size
constexpr int kThreads = 256;
constexpr int kTile = kC * kN * 2;     // bytes of one bf16 64x64 tile
constexpr int kStages = 2;
constexpr int kStageBytes = 4 * kTile; // r, k, v, w
constexpr float kHazard = 8.673617379884035e-19f;  // 2^-60

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_STAGE = 0;                          // stage s: R | K | V | W
constexpr int SLOT_R = 0, SLOT_K = kTile, SLOT_V = 2 * kTile, SLOT_W = 3 * kTile;
constexpr int OFF_KB = kStages * kStageBytes;         // Kb tile
constexpr int OFF_QI = OFF_KB + kTile;                // Qi tile
constexpr int OFF_QO = OFF_QI + kTile;                // Qo_0 at +0, Qo_1 at +4096, Qo_2 at +8192
constexpr int OFF_SMALL = OFF_QO + 2 * kTile;         // fp32 scratch below
constexpr int OFF_H = OFF_SMALL;                      // [4][2][64] half-block totals
constexpr int OFF_D = OFF_H + 4 * 2 * 64 * 4;         // [64] chunk decay
constexpr int OFF_UB = OFF_D + 64 * 4;                // [64] bonus diagonal
constexpr int OFF_DD = OFF_UB + 64 * 4;               // [4][16][16] exact diagonal blocks
constexpr int OFF_BAR = OFF_DD + 4 * 16 * 16 * 4;     // mbarriers (8 bytes each)
constexpr int OFF_MISC = OFF_BAR + 8 * 8;             // tmem base, flags
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;      // + alignment slack

// TMEM columns (fp32 accumulators, M = 64 layout: row m -> lane (m % 16) + 32 (m / 16))
constexpr uint32_t COL_S = 0, COL_AD = 64, COL_AO = 128, COL_O = 192, kTmemCols = 256;

// ---------------------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// byte offset of (row, byte column) inside a 64-row x 128-byte tile with 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int row, int colbyte)
{
    return row * 128 + ((((colbyte >> 4) ^ (row & 7))) << 4) + (colbyte & 15);
}

// UMMA shared-memory descriptor: 128-byte swizzle, SBO = 1024 (8-row groups)
__device__ __forceinline__ uint64_t udesc(uint32_t addr, uint32_t lbo)
{
    return static_cast<uint64_t>((addr >> 4) & 0x3FFF) |
           (static_cast<uint64_t>((lbo >> 4) & 0x3FFF) << 16) |
           (static_cast<uint64_t>(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ uint64_t desc_k(uint32_t addr) { return udesc(addr, 16); }
__device__ __forceinline__ uint64_t desc_mn(uint32_t addr) { return udesc(addr, kTile); }

// instruction descriptor: bf16 x bf16 -> fp32, M = 64
__host__ __device__ constexpr uint32_t idesc(int n, int a_mn, int b_mn)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
           (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(n >> 3) << 17) |
           (static_cast<uint32_t>(64 >> 4) << 24);
}

__device__ __forceinline__ void mma(uint32_t d, uint64_t a, uint64_t b, uint32_t id, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
                 "l"(a), "l"(b), "r"(id), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ bool bar_try(uint32_t bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred P;\n\tmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, P;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(phase)
                 : "memory");
    return ok != 0;
}

// Bounded wait; returns false if the limit ran out.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t phase, uint32_t limit)
{
    for (uint32_t it = 0; it < limit; ++it)
        if (bar_try(bar, phase)) return true;
    return false;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// 16 TMEM lanes x 32 columns split in two halves: threads 0-15 get columns [c, c+16),
// threads 16-31 get [c+16, c+32), each thread one lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
                 "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
                 "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
                 "r"(__float_as_uint(v[15]))
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ float2 ld_bf2(const unsigned char *tile, uint32_t off)
{
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(tile + off));
}

__device__ __forceinline__ void st_bf2(unsigned char *tile, uint32_t off, float2 x)
{
    *reinterpret_cast<uint32_t *>(tile + off) = pack_bf16(x.x, x.y);
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return make_float2(a.x * b.x, a.y * b.y); }

// 16 consecutive fp32 of one row -> 32 bytes of bf16 at (row, colbyte) of a swizzled tile
__device__ __forceinline__ void st_row16_bf16(unsigned char *tile, int row, int colbyte, const float (&v)[16])
{
    uint4 a, b;
    a.x = pack_bf16(v[0], v[1]);
    a.y = pack_bf16(v[2], v[3]);
    a.z = pack_bf16(v[4], v[5]);
    a.w = pack_bf16(v[6], v[7]);
    b.x = pack_bf16(v[8], v[9]);
    b.y = pack_bf16(v[10], v[11]);
    b.z = pack_bf16(v[12], v[13]);
    b.w = pack_bf16(v[14], v[15]);
    *reinterpret_cast<uint4 *>(tile + swz(row, colbyte)) = a;
    *reinterpret_cast<uint4 *>(tile + swz(row, colbyte + 16)) = b;
}

struct ChunkedParams {
    int64_t T, H;
    const float *u, *s0;
    __nv_bfloat16 *y;
    float *sT;
    int *status;
    uint32_t spin_limit;
    int inject_timeout;
};

__global__ void __launch_bounds__(kThreads, 2)
wkv6_chunked_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                    const ChunkedParams p)
{
    extern __shared__ unsigned char smem_raw[];
    unsigned char *sm = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    float *Hs = reinterpret_cast<float *>(sm + OFF_H);
    float *Dv = reinterpret_cast<float *>(sm + OFF_D);
    float *UB = reinterpret_cast<float *>(sm + OFF_UB);
    float *DD = reinterpret_cast<float *>(sm + OFF_DD);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(sm + OFF_MISC);
    // bars: 0,1 = stage full; 2 = scores done; 3 = chunk MMAs done; 4 = never arrived (test hook)
    const uint32_t bar_full0 = smem_u32(&bars[0]);
    const uint32_t bar_A = smem_u32(&bars[2]);
    const uint32_t bar_O = smem_u32(&bars[3]);
    const uint32_t bar_never = smem_u32(&bars[4]);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / p.H, h = bh % p.H;
    const int64_t T = p.T;
    const int nchunks = static_cast<int>((T + kC - 1) / kC);
    const uint32_t limit = p.spin_limit;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) bar_init(bar_full0 + 8 * s, 1);
        bar_init(bar_A, 1);
        bar_init(bar_O, 1);
        bar_init(bar_never, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(const_cast<uint32_t *>(misc))),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tbase = misc[0];

    // TMA issue for one chunk into its stage (thread 0 only)
    auto issue = [&](int c) {
        const int s = c % kStages;
        const uint32_t dst = smem_u32(sm + OFF_STAGE + s * kStageBytes);
        const uint32_t bar = bar_full0 + 8 * s;
        bar_expect_tx(bar, kStageBytes);
        const int t0 = c * kC;
        tma_load_4d(dst + SLOT_R, &map_r, 0, static_cast<int>(h), t0, static_cast<int>(b), bar);
        tma_load_4d(dst + SLOT_K, &map_k, 0, static_cast<int>(h), t0, static_cast<int>(b), bar);
        tma_load_4d(dst + SLOT_V, &map_v, 0, static_cast<int>(h), t0, static_cast<int>(b), bar);
        tma_load_4d(dst + SLOT_W, &map_w, 0, static_cast<int>(h), t0, static_cast<int>(b), bar);
    };
    int issued = 0;  // chunks issued so far (thread 0)
    if (tid == 0) {
        for (; issued < kStages && issued < nchunks; ++issued) issue(issued);
    }

    // warp roles for the TMEM passes: lane quadrant q (rows 16q..16q+15), column half ch
    const int q = warp & 3, ch = warp >> 2, hi = lane >> 4, lr = lane & 15;
    const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * q) << 16);
    const int row = 16 * q + lr;          // TMEM row served by this thread
    const int col0 = 32 * ch + 16 * hi;   // first of its 16 columns

    // initial state into TMEM
    {
        float v[16];
        if (p.s0) {
            const float4 *src = reinterpret_cast<const float4 *>(p.s0 + (bh * kN + row) * kN + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float4 x = src[i];
                v[4 * i] = x.x;
                v[4 * i + 1] = x.y;
                v[4 * i + 2] = x.z;
                v[4 * i + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = 0.f;
        }
        tmem_st16(tlane + COL_S + 32 * ch, v);
    }

    // prep roles: sub-block a, half hf, channel pair cp
    const int pa = warp >> 1, phf = warp & 1, cp = lane;
    const float2 u2 = *reinterpret_cast<const float2 *>(p.u + h * kN + 2 * cp);

    int abort = 0;
    if (p.inject_timeout && tid == 0) abort = !bar_wait(bar_never, 0, limit);
    fence_before();
    abort = __syncthreads_or(abort);
    fence_after();
    if (abort) record_status(p.status, kStatusTimeout);

    int c = 0;
    for (; c < nchunks && !abort; ++c) {
        const int s = c % kStages;
        unsigned char *st = sm + OFF_STAGE + s * kStageBytes;
        const int t0 = c * kC;
        const int tv = static_cast<int>(T - t0 < kC ? T - t0 : kC);
        int ok = bar_wait(bar_full0 + 8 * s, (c / kStages) & 1, limit);

        // ---- prep step 1: running products within this thread's 8-token half block
        float2 rr[8], kk[8], ww[8], pre[8], suf[8];
        const int tb0 = 16 * pa + 8 * phf;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            const int t = tb0 + m;
            const uint32_t off = swz(t, 4 * cp);
            if (t < tv) {
                rr[m] = ld_bf2(st + SLOT_R, off);
                kk[m] = ld_bf2(st + SLOT_K, off);
                ww[m] = ld_bf2(st + SLOT_W, off);
            } else {
                rr[m] = make_float2(0.f, 0.f);
                kk[m] = make_float2(0.f, 0.f);
                ww[m] = make_float2(1.f, 1.f);
            }
        }
        float2 run = make_float2(1.f, 1.f);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            pre[m] = run;
            run = mul2(run, ww[m]);
        }
        const float2 Hhalf = run;
        run = make_float2(1.f, 1.f);
#pragma unroll
        for (int m = 7; m >= 0; --m) {
            suf[m] = run;
            run = mul2(run, ww[m]);
        }
        // bonus diagonal sum_c r u k per token (reduce over the warp's 64 channels)
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            float part = rr[m].x * u2.x * kk[m].x + rr[m].y * u2.y * kk[m].y;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == m) UB[tb0 + m] = part;
        }
        *reinterpret_cast<float2 *>(Hs + (pa * 2 + phf) * 64 + 2 * cp) = Hhalf;
        if (__syncthreads_or(!ok)) {
            abort = 1;
            break;
        }

        // ---- sub-block totals, hazard check
        float2 G[4];
#pragma unroll
        for (int be = 0; be < 4; ++be)
            G[be] = mul2(*reinterpret_cast<const float2 *>(Hs + (be * 2 + 0) * 64 + 2 * cp),
                         *reinterpret_cast<const float2 *>(Hs + (be * 2 + 1) * 64 + 2 * cp));
        int hazard_local = 0;
#pragma unroll
        for (int be = 0; be < 4; ++be) hazard_local |= (G[be].x < kHazard) | (G[be].y < kHazard);
        const int hazard = __syncthreads_or(hazard_local);

        if (hazard) {
            // exact diagonal blocks from running products (inputs are still intact here)
            for (int item = tid; item < 4 * 120; item += kThreads) {
                const int ab = item / 120;
                int pr = item % 120, tt = 1;
                while (pr >= tt) {
                    pr -= tt;
                    ++tt;
                }
                const int ii = pr;  // 0 <= ii < tt < 16
                const int t = 16 * ab + tt, i = 16 * ab + ii;
                float acc = 0.f;
                if (t < tv) {
                    for (int cc = 0; cc < kN; cc += 2) {
                        const float2 rt = ld_bf2(st + SLOT_R, swz(t, 2 * cc));
                        const float2 ki = ld_bf2(st + SLOT_K, swz(i, 2 * cc));
                        float2 f = make_float2(1.f, 1.f);
                        for (int j = i + 1; j < t; ++j) f = mul2(f, ld_bf2(st + SLOT_W, swz(j, 2 * cc)));
                        acc += rt.x * ki.x * f.x + rt.y * ki.y * f.y;
                    }
                }
                DD[(ab * 16 + tt) * 16 + ii] = acc;
            }
            __syncthreads();
        }

        // ---- prep step 2: operand tiles (Qd -> R slot, Kd -> K slot, Kh -> W slot in place)
        {
            const float2 one = make_float2(1.f, 1.f);
            const float2 Hb0 = *reinterpret_cast<const float2 *>(Hs + (pa * 2 + 0) * 64 + 2 * cp);
            const float2 Hb1 = *reinterpret_cast<const float2 *>(Hs + (pa * 2 + 1) * 64 + 2 * cp);
            const float2 lead = phf ? Hb0 : one;
            const float2 trail = phf ? one : Hb1;
            float2 before = one, after = one;
#pragma unroll
            for (int be = 0; be < 4; ++be) {
                if (be < pa) before = mul2(before, G[be]);
                if (be > pa) after = mul2(after, G[be]);
            }
            // C_{a,b} = prod_{beta=b+1}^{a-1} G_beta for b = a-1, a-2, a-3
            float2 cab[3];
            cab[0] = one;                          // b = a-1
            cab[1] = pa >= 2 ? G[pa - 1] : one;    // b = a-2
            cab[2] = pa >= 3 ? mul2(G[pa - 2], G[pa - 1]) : one;  // b = a-3
            unsigned char *qo = sm + OFF_QO;
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int t = tb0 + m;
                const uint32_t off = swz(t, 4 * cp);
                const float2 pex = mul2(lead, pre[m]);
                const float2 pin = mul2(pex, ww[m]);
                const float2 sex = mul2(suf[m], trail);
                const float2 qd = mul2(rr[m], pex);
                float2 kd;
                kd.x = pin.x >= kHazard ? kk[m].x * rcp_approx(pin.x) : 0.f;
                kd.y = pin.y >= kHazard ? kk[m].y * rcp_approx(pin.y) : 0.f;
                const float2 kb = mul2(kk[m], sex);
                st_bf2(st + SLOT_R, off, qd);
                st_bf2(st + SLOT_K, off, kd);
                st_bf2(sm + OFF_KB, off, kb);
                st_bf2(sm + OFF_QI, off, mul2(qd, before));
                st_bf2(st + SLOT_W, off, mul2(kb, after));
#pragma unroll
                for (int d = 1; d <= 3; ++d) {
                    if (d <= pa) {
                        const int bq = pa - d;  // key sub-block served by Qo_bq
                        st_bf2(qo + 4096 * bq, off, mul2(qd, cab[d - 1]));
                    }
                }
            }
            if (warp == 0) {
                float2 D = one;
#pragma unroll
                for (int be = 0; be < 4; ++be) D = mul2(D, G[be]);
                *reinterpret_cast<float2 *>(Dv + 2 * cp) = D;
            }
        }
        fence_async_smem();
        fence_before();
        __syncthreads();
        fence_after();

        // ---- scores: diagonal (N=64) and off-diagonal (3 x N=16) MMAs
        if (tid == 0) {
            const uint32_t aR = smem_u32(st + SLOT_R), aK = smem_u32(st + SLOT_K);
            const uint32_t aKB = smem_u32(sm + OFF_KB), aQO = smem_u32(sm + OFF_QO);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma(tbase + COL_AD, desc_k(aR + 32 * ks), desc_k(aK + 32 * ks), idesc(64, 0, 0), ks > 0);
#pragma unroll
            for (int bq = 0; bq < 3; ++bq)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma(tbase + COL_AO + 16 * bq, desc_k(aQO + 4096 * bq + 32 * ks),
                        desc_k(aKB + 2048 * bq + 32 * ks), idesc(16, 0, 0), ks > 0);
            mma_commit(bar_A);
        }
        ok = bar_wait(bar_A, c & 1, limit);
        fence_after();

        // ---- mask pass: P (bf16, causal, bonus diagonal) -> K slot
        {
            float vd[16], vo[16], pv[16];
            tmem_ld16(tlane + COL_AD + 32 * ch, vd);
            tmem_ld16(tlane + COL_AO + 32 * ch, vo);
            const int kb = 2 * ch + hi;  // key sub-block of this thread's 16 columns
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                float val = 0.f;
                if (kb < q) {
                    val = vo[n];
                } else if (kb == q) {
                    if (n < lr) val = hazard ? DD[(q * 16 + lr) * 16 + n] : vd[n];
                    else if (n == lr) val = UB[row];
                }
                pv[n] = val;
            }
            st_row16_bf16(st + SLOT_K, row, 32 * kb, pv);
        }

        // ---- state pass: S_prev -> bf16 operand (R slot), S *= D in TMEM
        {
            float sv[16];
            tmem_ld16(tlane + COL_S + 32 * ch, sv);
            st_row16_bf16(st + SLOT_R, row, 2 * col0, sv);
            const float d = Dv[row];
#pragma unroll
            for (int n = 0; n < 16; ++n) sv[n] *= d;
            tmem_st16(tlane + COL_S + 32 * ch, sv);
        }
        fence_async_smem();
        fence_before();
        if (__syncthreads_or(!ok)) {
            abort = 1;
            break;
        }
        fence_after();

        // ---- O = P V + Qi S_prev ; S += Kh^T V
        if (tid == 0) {
            const uint32_t aP = smem_u32(st + SLOT_K), aV = smem_u32(st + SLOT_V);
            const uint32_t aSb = smem_u32(st + SLOT_R), aKh = smem_u32(st + SLOT_W);
            const uint32_t aQI = smem_u32(sm + OFF_QI);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma(tbase + COL_O, desc_k(aP + 32 * ks), desc_mn(aV + 2048 * ks), idesc(64, 0, 1), ks > 0);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma(tbase + COL_O, desc_k(aQI + 32 * ks), desc_mn(aSb + 2048 * ks), idesc(64, 0, 1), 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma(tbase + COL_S, desc_mn(aKh + 2048 * ks), desc_mn(aV + 2048 * ks), idesc(64, 1, 1), 1);
            mma_commit(bar_O);
        }
        ok = bar_wait(bar_O, c & 1, limit);
        fence_after();

        // stage is free: prefetch the chunk that reuses it
        if (tid == 0 && ok && issued < nchunks) {
            issue(issued);
            ++issued;
        }

        // ---- epilogue: O -> y (bf16)
        {
            float ov[16];
            tmem_ld16(tlane + COL_O + 32 * ch, ov);
            if (row < tv) {
                uint4 a, bb;
                a.x = pack_bf16(ov[0], ov[1]);
                a.y = pack_bf16(ov[2], ov[3]);
                a.z = pack_bf16(ov[4], ov[5]);
                a.w = pack_bf16(ov[6], ov[7]);
                bb.x = pack_bf16(ov[8], ov[9]);
                bb.y = pack_bf16(ov[10], ov[11]);
                bb.z = pack_bf16(ov[12], ov[13]);
                bb.w = pack_bf16(ov[14], ov[15]);
                uint4 *dst = reinterpret_cast<uint4 *>(p.y + ((b * T + t0 + row) * p.H + h) * kN + col0);
                dst[0] = a;
                dst[1] = bb;
            }
        }
        fence_before();
        if (__syncthreads_or(!ok)) {
            abort = 1;
            break;
        }
        fence_after();
    }

    // ---- final state
    if (abort) record_status(p.status, kStatusTimeout);
    if (!abort) {
        if (p.sT) {
            float sv[16];
            tmem_ld16(tlane + COL_S + 32 * ch, sv);
            float4 *dst = reinterpret_cast<float4 *>(p.sT + (bh * kN + row) * kN + col0);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                dst[i] = make_float4(sv[4 * i], sv[4 * i + 1], sv[4 * i + 2], sv[4 * i + 3]);
        }
    } else if (tid == 0) {
        // abort: wait (bounded) for this CTA's own copies and MMAs before releasing memory
        for (int cc = c; cc < issued; ++cc) bar_wait(bar_full0 + 8 * (cc % kStages), (cc / kStages) & 1, limit);
        mma_commit(bar_never);
        bar_wait(bar_never, 0, limit);
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *ptr = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// [B, T, H, N] bf16, box = 64 channels x 1 head x 64 tokens x 1 batch row
bool make_map(CUtensorMap *map, const void *base, int64_t B, int64_t T, int64_t H)
{
    auto enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(kN), static_cast<cuuint64_t>(H),
                          static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {static_cast<cuuint64_t>(kN * 2), static_cast<cuuint64_t>(H * kN * 2),
                             static_cast<cuuint64_t>(T * H * kN * 2)};
    cuuint32_t box[4] = {kN, 1, kC, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides,
                     box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

int g_chunked_inject_timeout = 0;  // test hook: set through rwkv_debug_inject_timeout

cudaError_t wkv6_chunked_launch(const Wkv6Args &a, cudaStream_t s)
{
    if (!a.bf16) return wkv6_serial_launch(a, s);
    const int64_t blocks = a.B * a.H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL || a.T > 0x7fffffffLL - kC || a.B > 0x7fffffffLL || a.H > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    CUtensorMap mr, mk, mv, mw;
    if (!make_map(&mr, a.r, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mw, a.w, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(wkv6_chunked_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kSmemBytes);
    if (e != cudaSuccess) return e;
    ChunkedParams prm{a.T, a.H, a.u, a.s0, static_cast<__nv_bfloat16 *>(a.y), a.sT, a.status,
                      g_chunked_inject_timeout ? 20000u : (1u << 20), g_chunked_inject_timeout};
    wkv6_chunked_kernel<<<static_cast<unsigned>(blocks), kThreads, kSmemBytes, s>>>(mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

}  // namespace wkv
