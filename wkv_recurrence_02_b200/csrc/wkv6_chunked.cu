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
// One CTA owns one (batch row, head) -- or one segment of it when sequences are split --
// and walks its sequence in 64-token chunks.  The fp32 state S (64x64) lives in tensor
// memory for the whole sequence.  Per chunk, with every decay referenced to the chunk end
// (running products of w on CUDA cores -- no logarithms):
//
//   Qx[t] = r_t / prod_{j>=t} w_j      (written over the r tile)
//   Kh[i] = k_i * prod_{j>i} w_j       (written over the k tile; every factor <= 1)
//   A     = Qx Kh^T                    scores: A[t][i] = r_t . (k_i prod_{j=i+1}^{t-1} w_j)
//   P     = causal mask of A with the bonus sum_c r_t[c] u[c] k_t[c] on the diagonal (bf16)
//   O     = P V + Qx . bf16(D (.) S_prev)      (Qx (.) D = r_t prod_{j<t} w_j)
//   S     = diag(D) S_prev + Kh^T V,   D = prod_j w_j over the chunk
//
// If some channel's chunk decay D falls below 2^-100, 1/prod could overflow: that chunk
// takes the sub-block path instead, with each 16-token query sub-block referenced to its
// own start (all off-diagonal factors <= 1, three extra MMAs of N = 16 into TMEM), and the
// 16x16 diagonal blocks either factored about the sub-block start or, when a 16-token
// product is below 2^-60, computed exactly on CUDA cores.
//
// The products are tcgen05.mma kind::f16 (bf16 operands from 128-byte-swizzled shared
// memory, fp32 accumulators in TMEM); S_prev is read from TMEM into a bf16 operand tile.
// On the chunk-end path P is written back into tensor memory as bf16 pairs and the P V
// product takes its A operand from there.
// r, k, v, w tiles arrive by TMA (4-D tensor maps over [B, T, H, N], 128-byte swizzle,
// zero fill past T) into a 3-stage ring.
//
// Every mbarrier wait is bounded; on expiry the CTA records RWKV_ERR_TIMEOUT in the
// device status word, waits (bounded) for its own copies and MMAs, frees its tensor
// memory and returns.
#include "tc_common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>
#include <algorithm>
#include <mutex>

namespace wkv {
namespace {
using namespace tc;

constexpr int kC = 64;                 // tokens per chunk
constexpr int kN = 64;                 // head size
constexpr int kThreads = 256;
constexpr int kPrepThreads = 128;
constexpr int kStages = 3;
constexpr int kStageBytes = 4 * kTile; // r, k, v, w
constexpr float kHazard = 8.673617379884035e-19f;  // 2^-60: sub-block factor guard
constexpr float kFastMin = 7.888609052210118e-31f; // 2^-100: chunk-end reference guard

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int OFF_STAGE = 0;                          // stage s: R | K | V | W
constexpr int SLOT_R = 0, SLOT_K = kTile, SLOT_V = 2 * kTile, SLOT_W = 3 * kTile;
// A chunk on the sub-block path borrows the stage two chunks ahead as scratch:
constexpr int SCR_KB = 0, SCR_QI = kTile, SCR_QO = 2 * kTile;  // Qo_b at SCR_QO + 4096 b
// bf16 (D S_prev) operand of a chunk-end-path chunk.  A sub-block-path chunk keeps its state
// operand in its own stage instead and uses this tile for its [4][16][16] fp32 exact diagonal
// blocks (written once the previous chunk's products, the tile's last readers, are done).
constexpr int OFF_SB = kStages * kStageBytes;
constexpr int OFF_SMALL = OFF_SB + kTile;             // fp32 bookkeeping below
// [chunk parity][4][64] 16-token sub-block products: two buffers, so a prep warp that has
// moved on to the next chunk never overwrites products another warp is still reading
constexpr int OFF_H = OFF_SMALL;
constexpr int OFF_D = OFF_H + 2 * 4 * 64 * 4;         // [stage][64] chunk decay
constexpr int OFF_UB = OFF_D + kStages * 64 * 4;      // [stage][64] bonus diagonal
constexpr int OFF_BAR = OFF_UB + kStages * 64 * 4;    // mbarriers (8 bytes each)
constexpr int OFF_MISC = OFF_BAR + 16 * 8;            // tmem base, flags
constexpr int OFF_LN = OFF_MISC + 64;                 // [2][64] LayerNorm scale, shift of the head
constexpr int kSmemBytes = OFF_LN + 2 * 64 * 4 + 1024; // + alignment slack

// TMEM columns (fp32 accumulators, M = 64 layout: row m -> lane (m % 16) + 32 (m / 16))
constexpr uint32_t COL_S = 0, COL_AD = 64, COL_AO = 128, COL_O = 192, kTmemCols = 256;

struct ChunkedParams {
    int64_t T, H;
    const float *u, *s0;
    __nv_bfloat16 *y;
    float *sT;
    int *status;
    uint32_t spin_limit;
    int inject_timeout;
    // sequence split: CTA (bh, g) covers chunks [g * seg_chunks, (g + 1) * seg_chunks) and
    // starts from s0 carried over the pieces before it: `pieces` entries per segment of
    // (end state from zero, decay product) in seg, written by the first pass
    int seg_chunks;        // chunks per segment (>= number of chunks when not split)
    float *seg;            // [B*H][nsub][N*N + N]
    int nseg;              // segments per sequence
    int pieces;            // first-pass pieces per segment
    int nsub;              // first-pass pieces per sequence, (nseg - 1) * pieces
    int64_t seg_cap;       // floats of scratch behind seg (index checks of the debug build)
    // fused output stage (null gate: plain y): y = SiLU(g) (ln_w (o - mean) rstd + ln_b)
    const __nv_bfloat16 *gate;
    const float *ln_w, *ln_b;
    float eps;
};
constexpr int kSegStride = kN * kN + kN;

// TMA of chunk c (r, k, v, w tiles of one head) into its stage, one thread.
__device__ __forceinline__ void issue_chunk(unsigned char *sm, uint32_t bar_full0, const CUtensorMap *mr,
                                            const CUtensorMap *mk, const CUtensorMap *mv,
                                            const CUtensorMap *mw, int c, int cabs, int h, int b,
                                            int *status, int64_t T)
{
    const int s = c % kStages;  // c counts chunks within this CTA's segment
    // debug build: a tile starting past T is not issued (its wait then runs out)
    if (!tma_coord_ok(status, 0, 2, kN, static_cast<int64_t>(cabs) * kC, T)) return;
    if (!in_bounds(status, OFF_STAGE + s * kStageBytes, kStageBytes, OFF_SB)) return;
    const uint32_t dst = smem_u32(sm + OFF_STAGE + s * kStageBytes);
    const uint32_t bar = bar_full0 + 8 * s;
    bar_expect_tx(bar, kStageBytes);
    const int t0 = cabs * kC;
    tma_load_4d(dst + SLOT_R, mr, 0, h, t0, b, bar);
    tma_load_4d(dst + SLOT_K, mk, 0, h, t0, b, bar);
    tma_load_4d(dst + SLOT_V, mv, 0, h, t0, b, bar);
    tma_load_4d(dst + SLOT_W, mw, 0, h, t0, b, bar);
}

// Sum over the 16 lanes of a half-warp of 8 per-lane partials (one per token m = 0..7).
// Returns the total for token (lane >> 1) & 7 (valid in every lane).
__device__ __forceinline__ float half_sum8(const float (&part)[8], int lane)
{
    float v4[4], v2[2];
    const bool b8 = lane & 8, b4 = lane & 4, b2 = lane & 2;
#pragma unroll
    for (int i = 0; i < 4; ++i)
        v4[i] = (b8 ? part[4 + i] : part[i]) + __shfl_xor_sync(0xffffffffu, b8 ? part[i] : part[4 + i], 8);
#pragma unroll
    for (int i = 0; i < 2; ++i)
        v2[i] = (b4 ? v4[2 + i] : v4[i]) + __shfl_xor_sync(0xffffffffu, b4 ? v4[i] : v4[2 + i], 4);
    float v = (b2 ? v2[1] : v2[0]) + __shfl_xor_sync(0xffffffffu, b2 ? v2[0] : v2[1], 2);
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    return v;
}

// Chunk-end path operand rows of one 8-token half sub-block, four channels per thread:
// Qx -> R slot, Kh -> K slot, and the bonus partials.  FULL: all 8 tokens valid.
// 1 / prod_{j>=t} w_j is formed as (1/D) prod_{j<t} w_j: a forward running product from
// `pre` = (1/D) times the product of w before this half, one reciprocal per channel and
// chunk instead of one per element (on this path D >= 2^-100, so pre stays below 2^100).
template <bool FULL>
__device__ __forceinline__ void prep_fast(unsigned char *st, int t0h, uint32_t cbyte, int tv, const Q4 (&w)[8],
                                          Q4 after, Q4 pre, Q4 u, float (&part)[8])
{
    Q4 suf[8];  // product of w over the tokens after token m of this half, to the chunk end
    suf[7] = after;
#pragma unroll
    for (int m = 7; m >= 1; --m) suf[m - 1] = mul4(suf[m], w[m]);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const int t = t0h + m;
        const uint32_t off = swz(t, cbyte);
        uint2 rr = make_uint2(0u, 0u), kk = rr;
        if (FULL || t < tv) {
            rr = ld_u2(st + SLOT_R, off);
            kk = ld_u2(st + SLOT_K, off);
        }
        const Q4 r = unpack4(rr), k = unpack4(kk);
        st_u2(st + SLOT_R, off, pack4(mul4(r, pre)));
        st_u2(st + SLOT_K, off, pack4(mul4(k, suf[m])));
        part[m] = bonus4(r, u, k);
        pre = mul4(pre, w[m]);
    }
}

// y row of token tok, head h: this thread's 32 of the 64 channels, the other 32 in lane
// ^ 16.  With a gate, the head's LayerNorm (statistics over both halves) and the SiLU gate
// are applied first, in f32x2 pairs, and the gated branch stores the row itself.  Every lane of the warp calls this (the statistics pair lanes); only
// `valid` rows read g and store.
template <bool GATED>
__device__ __forceinline__ void store_y_row(const ChunkedParams &p, float (&ov)[32], int64_t tok, int64_t b,
                                            int64_t h, int colh, bool valid, const float *lns)
{
    // debug build: the row must be a token of the sequence and lie inside y (and g)
    valid = valid && in_bounds(p.status, tok, 1, p.T) &&
            in_bounds(p.status, ((b * p.T + tok) * p.H + h) * kN + colh, 32,
                      static_cast<int64_t>(gridDim.x) * p.T * kN);
    if (GATED) {
        uint4 gw[4] = {};  // the gate row, loaded first so that its latency overlaps the statistics
        if (valid) {
            const uint4 *gp = reinterpret_cast<const uint4 *>(p.gate + ((b * p.T + tok) * p.H + h) * kN + colh);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) gw[v4] = gp[v4];
        }
        // channel pairs in f32x2 registers: the statistics and the output stage take one
        // instruction per two channels
        P2 o2[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) o2[i] = pk(ov[2 * i], ov[2 * i + 1]);
        P2 sa = o2[0], sb = o2[1];
#pragma unroll
        for (int i = 2; i < 16; i += 2) {
            sa = add2(sa, o2[i]);
            sb = add2(sb, o2[i + 1]);
        }
        sa = add2(sa, sb);
        float s = lo(sa) + hi(sa);
        s += __shfl_xor_sync(0xffffffffu, s, 16);
        const float mean = s * (1.f / kN);
        const P2 nm = pk(-mean, -mean);
        P2 qa = pk(0.f, 0.f), qb = qa;
#pragma unroll
        for (int i = 0; i < 16; i += 2) {  // o2 now holds o - mean
            o2[i] = add2(o2[i], nm);
            o2[i + 1] = add2(o2[i + 1], nm);
            qa = fma2(o2[i], o2[i], qa);
            qb = fma2(o2[i + 1], o2[i + 1], qb);
        }
        qa = add2(qa, qb);
        float q = lo(qa) + hi(qa);
        q += __shfl_xor_sync(0xffffffffu, q, 16);
        const float rstd = rsqrtf(q * (1.f / kN) + p.eps);
        if (valid) {
            const P2 rs2 = pk(rstd, rstd), half2 = pk(0.5f, 0.5f);
            uint32_t yw[16];
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) {
                const uint32_t wd[4] = {gw[v4].x, gw[v4].y, gw[v4].z, gw[v4].w};
                // LayerNorm scale and shift of these 8 channels, 16-byte loads
                const float4 ca = *reinterpret_cast<const float4 *>(lns + colh + 8 * v4);
                const float4 cb = *reinterpret_cast<const float4 *>(lns + colh + 8 * v4 + 4);
                const float4 ha = *reinterpret_cast<const float4 *>(lns + kN + colh + 8 * v4);
                const float4 hb = *reinterpret_cast<const float4 *>(lns + kN + colh + 8 * v4 + 4);
                const P2 sc2[4] = {pk(ca.x, ca.y), pk(ca.z, ca.w), pk(cb.x, cb.y), pk(cb.z, cb.w)};
                const P2 sh2[4] = {pk(ha.x, ha.y), pk(ha.z, ha.w), pk(hb.x, hb.y), pk(hb.z, hb.w)};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const P2 hg = mul2(unpack2(wd[e]), half2);  // g / 2
                    const P2 t = fma2(mul2(sc2[e], o2[4 * v4 + e]), rs2, sh2[e]);
                    // SiLU(g) t = g sigma(g) t with sigma(g) = (1 + tanh(g/2)) / 2, i.e.
                    // (g t / 2)(1 + tanh(g / 2)): one approximate tanh per channel
                    const P2 x2 = mul2(hg, t);
                    yw[4 * v4 + e] = pack2(fma2(pk(tanh_approx(lo(hg)), tanh_approx(hi(hg))), x2, x2));
                }
            }
            // the stores last: a global store between them would hold back the shared loads of
            // the scale and shift, which the compiler cannot prove it does not alias
            uint4 *dst = reinterpret_cast<uint4 *>(p.y + ((b * p.T + tok) * p.H + h) * kN + colh);
#pragma unroll
            for (int v4 = 0; v4 < 4; ++v4) dst[v4] = make_uint4(yw[4 * v4], yw[4 * v4 + 1], yw[4 * v4 + 2], yw[4 * v4 + 3]);
        }
        return;
    }
    if (valid) {
        uint4 *dst = reinterpret_cast<uint4 *>(p.y + ((b * p.T + tok) * p.H + h) * kN + colh);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
            uint4 x;
            x.x = pack_bf16(ov[8 * v4 + 0], ov[8 * v4 + 1]);
            x.y = pack_bf16(ov[8 * v4 + 2], ov[8 * v4 + 3]);
            x.z = pack_bf16(ov[8 * v4 + 4], ov[8 * v4 + 5]);
            x.w = pack_bf16(ov[8 * v4 + 6], ov[8 * v4 + 7]);
            dst[v4] = x;
        }
    }
}

// Warp roles (256 threads):
//   warps 0-3  prep group: warp a builds the operand rows of 16-token sub-block a, running
//              up to two chunks ahead of the TMEM group;
//   warps 4-7  TMEM group: warp 4+q serves TMEM lanes of rows 16q..16q+15 (two 32-column
//              halves per warp); it writes y of chunk c-1 and builds P and the state operand
//              of chunk c in one pass.  In the full pass one elected thread of warp 4 issues
//              the O products, of warp 5 the state update, of warp 6 the next chunk's scores
//              (an MMA issue holds its thread for tens of cycles, so three issuers run side
//              by side), and of warp 7 the TMA copies of later chunks.
// Hand-offs are mbarriers: stage full (TMA -> prep), prep done (prep -> MMA issue), scores
// done, O done, state done and stage empty (tcgen05.commit).  Every TMEM thread waits on the
// scores, O and state barriers itself, and the TMEM group meets once per chunk, after its
// pass, before the products are issued.  Per-chunk bookkeeping (bonus diagonal, decay, path
// flags) lives beside the chunk's stage.
template <bool GATED, bool OMEGA>
__global__ void __launch_bounds__(kThreads, 2)
wkv6_chunked_kernel(const __grid_constant__ CUtensorMap map_r, const __grid_constant__ CUtensorMap map_k,
                    const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_w,
                    const ChunkedParams p)
{
    extern __shared__ unsigned char smem_raw[];
    // aligned by an offset on the __shared__ array itself (not through an integer), so the
    // compiler keeps the shared state space: its accesses are shared loads and stores, which it
    // may reorder freely around global ones
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    float *Hs2 = reinterpret_cast<float *>(sm + OFF_H);  // [parity][4 sub-blocks][64 channels]
    float *Dv = reinterpret_cast<float *>(sm + OFF_D);   // [stage][64]
    float *UB = reinterpret_cast<float *>(sm + OFF_UB);  // [stage][64]
    float *lns = reinterpret_cast<float *>(sm + OFF_LN);  // gated output: [scale, shift][64]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(sm + OFF_MISC);
    // misc: [0] TMEM base, [1] abort, [2+s] sub-block path, [5+s] exact diagonal (s = stage),
    //       [8] chunks whose TMA has been issued
    const uint32_t bar_full0 = smem_u32(&bars[0]);   // + 8 * stage
    const uint32_t bar_prep0 = smem_u32(&bars[3]);   // + 8 * stage
    const uint32_t bar_A = smem_u32(&bars[6]);
    const uint32_t bar_O = smem_u32(&bars[7]);
    const uint32_t bar_never = smem_u32(&bars[8]);
    const uint32_t bar_S = smem_u32(&bars[9]);
    const uint32_t bar_empty0 = smem_u32(&bars[10]);  // + 8 * stage: the chunk's MMAs are done
    const uint32_t bar_drain = smem_u32(&bars[13]);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / p.H, h = bh % p.H;
    const int64_t T = p.T;
    const int nchunks_all = static_cast<int>((T + kC - 1) / kC);
    // segment of the sequence; the last segments, which first combine the most pieces into
    // their incoming state, are dispatched first
    const int g = static_cast<int>(gridDim.y) - 1 - static_cast<int>(blockIdx.y);
    const int cb = g * p.seg_chunks;               // its first chunk
    const int nchunks = min(p.seg_chunks, nchunks_all - cb);  // chunks in this segment
    const uint32_t limit = p.spin_limit;
    const uint32_t spin_limit = p.spin_limit * 64u;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(bar_full0 + 8 * s, 1);
            bar_init(bar_prep0 + 8 * s, 128);
            bar_init(bar_empty0 + 8 * s, 2);  // O issuer and S issuer each commit
        }
        bar_init(bar_S, 1);
        bar_init(bar_drain, 3);
        bar_init(bar_A, 1);
        bar_init(bar_O, 1);
        bar_init(bar_never, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        misc[1] = 0;
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

    if (tid == 0) {
        int n0 = 0;
        for (; n0 < kStages - 1 && n0 < nchunks; ++n0)
            issue_chunk(sm, bar_full0, &map_r, &map_k, &map_v, &map_w, n0, cb + n0, static_cast<int>(h),
                        static_cast<int>(b), p.status, T);
        misc[8] = n0;
    }

    int abort = 0;
    if (p.inject_timeout && tid == 0) abort = !bar_wait(bar_never, 0, limit);
    abort = __syncthreads_or(abort);
    if (abort) misc[1] = 1;

    if (warp < 4) {
        // =============================== prep group ===============================
        // warp a: 16-token sub-block a; lane: half hf (tokens 16a + 8hf .. +7) and channel
        // quad cq (channels 4cq .. 4cq+3)
        const int a = warp, hf = lane >> 4, cq = lane & 15;
        const int t0h = 16 * a + 8 * hf;
        const uint32_t cbyte = 8 * cq;
        const Q4 u4 = in_bounds(p.status, h * kN + 4 * cq, 4, p.H * kN) ? ld_q4(p.u + h * kN + 4 * cq) : one4();
        for (int c = 0; c < nchunks && !abort; ++c) {
            const int s = c % kStages;
            unsigned char *st = sm + OFF_STAGE + s * kStageBytes;
            const int64_t t0 = static_cast<int64_t>(cb + c) * kC;
            const int tv = static_cast<int>(T - t0 < kC ? T - t0 : kC);
            // every thread waits for the stage itself (a group barrier here would hold all four
            // warps until the slowest has seen the data); a timeout is voted on at the barrier
            // below, where the whole group meets anyway
            int ok = bar_wait_spin(bar_full0 + 8 * s, (c / kStages) & 1, spin_limit);
            float *Hs = Hs2 + (c & 1) * 4 * 64;
            // w of this half (1.0 past the end) and its product; the other half's product
            Q4 w[8];
            Q4 Gh = one4();
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const int t = t0h + m;
                if (t < tv) {
                    const Q4 x = unpack4(ld_u2(st + SLOT_W, swz(t, cbyte)));
                    w[m] = OMEGA ? decay4(x) : x;
                } else {
                    w[m] = one4();
                }
                Gh = mul4(Gh, w[m]);
            }
            const Q4 Go = shfl_xor4(Gh, 16);
            if (hf == 0) st_q4(Hs + a * 64 + 4 * cq, mul4(Gh, Go));
            if (named_sync_or(1, 128, !ok || misc[1])) {
                abort = 1;
                misc[1] = 1;
                break;
            }
            // sub-block products from shared memory (read by index there: a register array
            // indexed by the warp's sub-block would be placed in local memory)
            Q4 D = one4(), before = one4(), aft = one4();
#pragma unroll
            for (int be = 0; be < 4; ++be) {
                const Q4 g = ld_q4(Hs + be * 64 + 4 * cq);
                D = mul4(D, g);
                before = be < a ? mul4(before, g) : before;
                aft = be > a ? mul4(aft, g) : aft;
            }
            // products over the tokens after this half (to the chunk end), from the
            // sub-block start to this half, and from this half's end to the sub-block end
            const Q4 after = hf ? aft : mul4(aft, Go);
            const Q4 lead = hf ? Go : one4(), trail = hf ? one4() : Go;
            // single chunk-end reference unless a chunk decay product is below 2^-100.  Every
            // warp's 32 lanes cover all 16 channel quads, so a warp vote is the chunk's vote
            // (the same in all four warps): no group barrier.
            const int safe = __any_sync(0xffffffffu, any_below(D, kFastMin));
            int hazard = 0;
            float part[8];
            if (!safe) {
                const Q4 pre = mul4({rcp2(D.a), rcp2(D.b)}, mul4(before, lead));
                if (tv == kC) prep_fast<true>(st, t0h, cbyte, tv, w, after, pre, u4, part);
                else prep_fast<false>(st, t0h, cbyte, tv, w, after, pre, u4, part);
            } else {
                // sub-block path; scratch = the stage two chunks ahead, free once chunk c-1 is done
                unsigned char *scr = sm + OFF_STAGE + ((c + 2) % kStages) * kStageBytes;
                // chunk c-1's stage, its ((c-1)/3)-th use
                if (c > 0 && tid == 0)
                    ok = bar_wait_spin(bar_empty0 + 8 * ((c + 2) % kStages), ((c - 1) / kStages) & 1, spin_limit);
                int hz = 0;
#pragma unroll
                for (int be = 0; be < 4; ++be) hz |= any_below(ld_q4(Hs + be * 64 + 4 * cq), kHazard);
                // C_{a,a-2}: product of sub-block a-1; C_{a,a-3}: of sub-blocks a-2 and a-1
                const Q4 cab1 = a >= 1 ? ld_q4(Hs + (a - 1) * 64 + 4 * cq) : one4();
                const Q4 cab2 = a >= 2 ? mul4(cab1, ld_q4(Hs + (a - 2) * 64 + 4 * cq)) : cab1;
                const int vote = __any_sync(0xffffffffu, hz);  // all channels, as above
                if (named_sync_or(1, 128, !ok)) {
                    abort = 1;
                    misc[1] = 1;
                    break;
                }
                if (c > 0) bar_try(bar_empty0 + 8 * ((c + 2) % kStages), ((c - 1) / kStages) & 1);
                hazard = vote;
                if (hazard) {
                    // exact diagonal blocks from running products (inputs still intact here)
                    const float2 one = make_float2(1.f, 1.f);
                    for (int item = tid; item < 4 * 120; item += 128) {
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
                                float2 f = one;
                                for (int j = i + 1; j < t; ++j) {
                                    float2 wj = ld_bf2(st + SLOT_W, swz(j, 2 * cc));
                                    if (OMEGA) wj = make_float2(decay_of_logit(wj.x), decay_of_logit(wj.y));
                                    f = mul2(f, wj);
                                }
                                acc += rt.x * ki.x * f.x + rt.y * ki.y * f.y;
                            }
                        }
                        reinterpret_cast<float *>(sm + OFF_SB)[(ab * 16 + tt) * 16 + ii] = acc;
                    }
                    named_sync_or(1, 128, 0);
                }
                // suf[m]: product of w from token m+1 of this half to the sub-block end
                Q4 suf[8];
                Q4 run = trail;
#pragma unroll
                for (int m = 7; m >= 0; --m) {
                    suf[m] = run;
                    run = mul4(run, w[m]);
                }
                Q4 pex = lead;  // product of w from the sub-block start to the token before t
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int t = t0h + m;
                    const uint32_t off = swz(t, cbyte);
                    uint2 rr = make_uint2(0u, 0u), kk = rr;
                    if (t < tv) {
                        rr = ld_u2(st + SLOT_R, off);
                        kk = ld_u2(st + SLOT_K, off);
                    }
                    const Q4 r = unpack4(rr), k = unpack4(kk);
                    const Q4 pin = mul4(pex, w[m]);
                    const Q4 qd = mul4(r, pex);
                    const Q4 kinv = {rcp2(pin.a), rcp2(pin.b)};
                    Q4 kd = mul4(k, kinv);
                    // Kd is dropped where the in-block product underflows the guard
                    kd.a = pk(lo(pin.a) >= kHazard ? lo(kd.a) : 0.f, hi(pin.a) >= kHazard ? hi(kd.a) : 0.f);
                    kd.b = pk(lo(pin.b) >= kHazard ? lo(kd.b) : 0.f, hi(pin.b) >= kHazard ? hi(kd.b) : 0.f);
                    const Q4 kbv = mul4(k, suf[m]);
                    st_u2(st + SLOT_R, off, pack4(qd));
                    st_u2(st + SLOT_K, off, pack4(kd));
                    st_u2(scr + SCR_KB, off, pack4(kbv));
                    st_u2(scr + SCR_QI, off, pack4(mul4(qd, before)));
                    st_u2(st + SLOT_W, off, pack4(mul4(kbv, aft)));
                    if (a >= 1) st_u2(scr + SCR_QO + 4096 * (a - 1), off, pack4(qd));              // Qo_{a-1}
                    if (a >= 2) st_u2(scr + SCR_QO + 4096 * (a - 2), off, pack4(mul4(qd, cab1)));  // Qo_{a-2}
                    if (a >= 3) st_u2(scr + SCR_QO + 4096 * (a - 3), off, pack4(mul4(qd, cab2)));  // Qo_{a-3}
                    part[m] = bonus4(r, u4, k);
                    pex = pin;
                }
            }
            const float tot = half_sum8(part, lane);
            if ((lane & 1) == 0) UB[s * 64 + t0h + ((lane >> 1) & 7)] = tot;
            if (warp == 0 && hf == 0) st_q4(Dv + s * 64 + 4 * cq, D);
            if (tid == 0) {
                misc[2 + s] = safe;
                misc[5 + s] = hazard;
            }
            fence_async_smem();
            bar_arrive(bar_prep0 + 8 * s);
        }
    } else {
        // =============================== TMEM group ===============================
        const int q = warp - 4, hi = lane >> 4, lr = lane & 15;
        const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * q) << 16);
        const int row = 16 * q + lr;   // TMEM row of this thread
        const int colh = 32 * hi;      // its 32 columns start here
        // one elected thread per warp: 4 issues the O products, 5 the state update, 6 the
        // scores of the next chunk (MMA issue blocks the issuing thread, so three issuers run
        // side by side), 7 the TMA copies
        const bool issuer = tid == kPrepThreads;
        const bool iss_o = issuer, iss_s = tid == kPrepThreads + 32, iss_a = tid == kPrepThreads + 64;
        const bool iss_t = tid == kPrepThreads + 96;
        int issued = misc[8];
        if (GATED) {  // the head's LayerNorm scale and shift (read after the loop's first barrier)
            const int t = tid - kPrepThreads;
            if (in_bounds(p.status, h * kN + (t & (kN - 1)), 1, p.H * kN))
                lns[t] = t < kN ? p.ln_w[h * kN + t] : p.ln_b[h * kN + t - kN];
        }

        // scores of chunk c into TMEM (issuer only)
        auto issue_scores = [&](int c) -> int {
            const int s = c % kStages;
            if (!bar_wait_spin(bar_prep0 + 8 * s, (c / kStages) & 1, spin_limit)) return 0;
            fence_after();
            unsigned char *st = sm + OFF_STAGE + s * kStageBytes;
            const uint32_t aR = smem_u32(st + SLOT_R), aK = smem_u32(st + SLOT_K);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                mma(tbase + COL_AD, desc_k(aR + 32 * ks), desc_k(aK + 32 * ks), idesc(64, 0, 0), ks > 0);
            if (misc[2 + s]) {
                // these columns hold the previous chunk's P when that chunk took the chunk-end
                // path: its O product must have read them first
                if (c > 0 && !misc[2 + (c - 1) % kStages] && !bar_wait_spin(bar_O, (c - 1) & 1, spin_limit))
                    return 0;
                unsigned char *scr = sm + OFF_STAGE + ((c + 2) % kStages) * kStageBytes;
                const uint32_t aKB = smem_u32(scr + SCR_KB), aQO = smem_u32(scr + SCR_QO);
#pragma unroll
                for (int bq = 0; bq < 3; ++bq)
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma(tbase + COL_AO + 16 * bq, desc_k(aQO + 4096 * bq + 32 * ks),
                            desc_k(aKB + 2048 * bq + 32 * ks), idesc(16, 0, 0), ks > 0);
            }
            mma_commit(bar_A);
            return 1;
        };

        int ok = 1;
        if (iss_a && !abort) ok = issue_scores(0);
        const int64_t nstate = static_cast<int64_t>(gridDim.x) * kN * kN;  // floats of s0 / sT
        // debug build: TMEM columns of this thread inside the allocation
        in_bounds(p.status, COL_O + colh, 32, kTmemCols);
        {   // initial state into TMEM: s0 carried over the pieces before this segment
            float v[32];
            if (p.s0 && in_bounds(p.status, (bh * kN + row) * kN + colh, 32, nstate)) {
                const float4 *src = reinterpret_cast<const float4 *>(p.s0 + (bh * kN + row) * kN + colh);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float4 x = src[i];
                    v[4 * i] = x.x;
                    v[4 * i + 1] = x.y;
                    v[4 * i + 2] = x.z;
                    v[4 * i + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            for (int gp = 0; gp < g * p.pieces; ++gp) {  // S <- diag(D_piece) S + S_piece
                if (!in_bounds(p.status, (bh * p.nsub + gp) * kSegStride, kSegStride, p.seg_cap)) break;
                const float *sg = p.seg + (bh * p.nsub + gp) * kSegStride;
                const float d = sg[kN * kN + row];
                const float4 *src = reinterpret_cast<const float4 *>(sg + row * kN + colh);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 x = src[i];
                    v[4 * i] = fmaf(d, v[4 * i], x.x);
                    v[4 * i + 1] = fmaf(d, v[4 * i + 1], x.y);
                    v[4 * i + 2] = fmaf(d, v[4 * i + 2], x.z);
                    v[4 * i + 3] = fmaf(d, v[4 * i + 3], x.w);
                }
            }
            tmem_st32(tlane + COL_S, v);
        }

        for (int c = 0; c < nchunks && !abort; ++c) {
            const int s = c % kStages;
            unsigned char *st = sm + OFF_STAGE + s * kStageBytes;
            const int64_t t0 = static_cast<int64_t>(cb + c) * kC;

            // scores of c and all MMAs of c-1 complete: every thread waits itself, so each warp
            // starts its pass as soon as they are; an expiry is voted on at the group barrier
            // after the pass (the warps must not leave the loop on their own)
            if (ok) ok = bar_wait_spin(bar_A, c & 1, spin_limit);
            if (ok && c > 0) ok = bar_wait_spin(bar_O, (c - 1) & 1, spin_limit);
            if (ok && c > 0) ok = bar_wait_spin(bar_S, (c - 1) & 1, spin_limit);
            bar_try(bar_prep0 + 8 * s, (c / kStages) & 1);  // the prep group's writes are visible
            fence_after();
            const int safe = misc[2 + s], hazard = misc[5 + s];

            // TMA for later chunks: a stage is free once its previous chunk is done, unless a
            // sub-block-path chunk still uses it as scratch
            if (iss_t) {
                while (issued < nchunks && issued <= c + kStages - 1) {
                    const int user = issued - 2;  // chunk that would use this stage as scratch
                    if (user >= c && misc[2 + user % kStages]) break;
                    issue_chunk(sm, bar_full0, &map_r, &map_k, &map_v, &map_w, issued, cb + issued,
                                static_cast<int>(h), static_cast<int>(b), p.status, T);
                    ++issued;
                }
                misc[8] = issued;
            }

            if (GATED) {  // the gate row of this thread's y row of chunk c (stored next iteration) into L2
                const int64_t tok = t0 + row;
                if (tok < T && in_bounds(p.status, ((b * T + tok) * p.H + h) * kN + colh, 32,
                                         static_cast<int64_t>(gridDim.x) * T * kN)) {
                    const __nv_bfloat16 *gp = p.gate + ((b * T + tok) * p.H + h) * kN + colh;
                    asm volatile("prefetch.global.L2 [%0];" ::"l"(gp));
                }
            }
            // ---- y of chunk c-1, and P of chunk c (causal scores, bonus diagonal, bf16)
            {
                if (c > 0) {
                    float ov[32];
                    tmem_ld32(tlane + COL_O, ov);
                    store_y_row<GATED>(p, ov, t0 - kC + row, b, h, colh, true, lns);
                }
                float va[32];
                tmem_ld32(tlane + COL_AD, va);
                if (safe) {
                    const float *DD = reinterpret_cast<const float *>(sm + OFF_SB);
                    float vo[32];
                    tmem_ld32(tlane + COL_AO, vo);
#pragma unroll
                    for (int n = 0; n < 32; ++n) {
                        const int kbi = (colh + n) >> 4;
                        if (kbi < q) va[n] = vo[n];
                        else if (kbi == q && hazard) va[n] = DD[(q * 16 + lr) * 16 + ((colh + n) & 15)];
                    }
                }
                // causal mask per 16-column block kb of this row: kb < q kept, kb == q the
                // diagonal block (columns before the row kept, the diagonal itself is the bonus
                // term), kb > q zero.  Chunk-end path: P goes to tensor memory, bf16 pairs in the
                // columns the sub-block path's scores use, and the O product reads it from there.
                if (!safe) {
                    const float ub = UB[s * 64 + row];
                    uint32_t pw[16];
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int kb = 2 * hi + j;
#pragma unroll
                        for (int n = 0; n < 16; n += 2) {
                            float x0 = va[16 * j + n], x1 = va[16 * j + n + 1];
                            if (kb > q) {
                                x0 = 0.f;
                                x1 = 0.f;
                            } else if (kb == q) {
                                x0 = n < lr ? x0 : (n == lr ? ub : 0.f);
                                x1 = n + 1 < lr ? x1 : (n + 1 == lr ? ub : 0.f);
                            }
                            pw[8 * j + n / 2] = pack_bf16(x0, x1);
                        }
                    }
                    tmem_st16w(tlane + COL_AO, pw);
                }
                unsigned char *pt = st + SLOT_K;
#pragma unroll
                for (int j = 0; j < 2 && safe; ++j) {
                    const int kb = 2 * hi + j;
                    float(&vb)[16] = *reinterpret_cast<float(*)[16]>(&va[16 * j]);
                    if (kb > q) {
                        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4 *>(pt + swz(row, 32 * kb)) = z;
                        *reinterpret_cast<uint4 *>(pt + swz(row, 32 * kb + 16)) = z;
                    } else {
                        if (kb == q) {
#pragma unroll
                            for (int n = 0; n < 16; ++n) vb[n] = n < lr ? vb[n] : 0.f;
                        }
                        st_row16_bf16(pt, row, 32 * kb, vb);
                    }
                }
                if (safe && hi == (q >> 1))  // the thread that holds the diagonal block
                    *reinterpret_cast<__nv_bfloat16 *>(pt + swz(row, 2 * row)) = __float2bfloat16_rn(UB[s * 64 + row]);
            }
            // ---- state: S *= D in TMEM; operand = bf16(D S_prev) (chunk-end path) or bf16(S_prev)
            {
                float sv[32];
                tmem_ld32(tlane + COL_S, sv);
                const float d = Dv[s * 64 + row];
                if (safe) {
                    st_row16_bf16(st + SLOT_R, row, 2 * colh, *reinterpret_cast<float(*)[16]>(&sv[0]));
                    st_row16_bf16(st + SLOT_R, row, 2 * colh + 32, *reinterpret_cast<float(*)[16]>(&sv[16]));
                }
#pragma unroll
                for (int n = 0; n < 32; ++n) sv[n] *= d;
                if (!safe) {
                    st_row16_bf16(sm + OFF_SB, row, 2 * colh, *reinterpret_cast<float(*)[16]>(&sv[0]));
                    st_row16_bf16(sm + OFF_SB, row, 2 * colh + 32, *reinterpret_cast<float(*)[16]>(&sv[16]));
                }
                tmem_st32(tlane + COL_S, sv);
            }
            fence_async_smem();
            fence_before();
            if (named_sync_or(2, 128, !ok || misc[1])) {
                abort = 1;
                misc[1] = 1;
                break;
            }
            fence_after();

            const uint32_t aV = smem_u32(st + SLOT_V);
            if (iss_o) {
                // ---- O = P V + Q S_op
                uint32_t aP = 0, aQ, aSop;
                if (!safe) {
                    aQ = smem_u32(st + SLOT_R);     // Qx
                    aSop = smem_u32(sm + OFF_SB);   // bf16(D S_prev)
                } else {
                    unsigned char *scr = sm + OFF_STAGE + ((c + 2) % kStages) * kStageBytes;
                    aP = smem_u32(st + SLOT_K);
                    aQ = smem_u32(scr + SCR_QI);    // Qi
                    aSop = smem_u32(st + SLOT_R);   // bf16(S_prev)
                }
                if (!safe) {  // P from tensor memory: 16 K elements are 8 columns
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma_ts(tbase + COL_O, tbase + COL_AO + 8 * ks, desc_mn(aV + 2048 * ks), idesc(64, 0, 1), ks > 0);
                } else {
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma(tbase + COL_O, desc_k(aP + 32 * ks), desc_mn(aV + 2048 * ks), idesc(64, 0, 1), ks > 0);
                }
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma(tbase + COL_O, desc_k(aQ + 32 * ks), desc_mn(aSop + 2048 * ks), idesc(64, 0, 1), 1);
                mma_commit(bar_O);
                mma_commit(bar_empty0 + 8 * s);
            } else if (iss_s) {
                // ---- S += Kh^T V  (Kh read MN-major as its transpose)
                const uint32_t aKh = smem_u32(st + (safe ? SLOT_W : SLOT_K));
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    mma(tbase + COL_S, desc_mn(aKh + 2048 * ks), desc_mn(aV + 2048 * ks), idesc(64, 1, 1), 1);
                mma_commit(bar_S);
                mma_commit(bar_empty0 + 8 * s);
            } else if (iss_a && c + 1 < nchunks) {
                ok = issue_scores(c + 1);  // scores of the next chunk
            }
        }
        // ---- y of the last chunk, and the final state
        if (!abort) {
            if (iss_o) ok = bar_wait_spin(bar_O, (nchunks - 1) & 1, spin_limit);
            else if (iss_s) ok = bar_wait_spin(bar_S, (nchunks - 1) & 1, spin_limit);
            if (named_sync_or(2, 128, !ok || misc[1])) {
                abort = 1;
                misc[1] = 1;
            } else {
                bar_try(bar_O, (nchunks - 1) & 1);
                bar_try(bar_S, (nchunks - 1) & 1);
                fence_after();
                float ov[32];
                tmem_ld32(tlane + COL_O, ov);
                const int64_t t0 = static_cast<int64_t>(cb + nchunks - 1) * kC;
                const int tv = static_cast<int>(T - t0 < kC ? T - t0 : kC);
                store_y_row<GATED>(p, ov, t0 + row, b, h, colh, row < tv, lns);
                if (p.sT && g == p.nseg - 1 && in_bounds(p.status, (bh * kN + row) * kN + colh, 32, nstate)) {
                    float sv[32];
                    tmem_ld32(tlane + COL_S, sv);
                    float4 *sd = reinterpret_cast<float4 *>(p.sT + (bh * kN + row) * kN + colh);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        sd[i] = make_float4(sv[4 * i], sv[4 * i + 1], sv[4 * i + 2], sv[4 * i + 3]);
                }
            }
        }
    }

    // ---- drain after an abort, then release tensor memory
    fence_before();
    abort = __syncthreads_or(abort | misc[1]);
    fence_after();
    if (abort) {
        record_status(p.status, kStatusTimeout);
        if (tid == kPrepThreads || tid == kPrepThreads + 32 || tid == kPrepThreads + 64) mma_commit(bar_drain);
        if (tid == kPrepThreads) {
            const int n = misc[8];
            for (int cc = n - kStages < 0 ? 0 : n - kStages; cc < n; ++cc)
                bar_wait(bar_full0 + 8 * (cc % kStages), (cc / kStages) & 1, limit);
            bar_wait(bar_drain, 0, limit);
        }
    }
    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(kTmemCols));
}

// ---------------------------------------------------------------------------- host side

}  // namespace

// [B, T, H, N] bf16, box = 64 channels x 1 head x 64 tokens x 1 batch row
bool make_map(CUtensorMap *map, const void *base, int64_t B, int64_t T, int64_t H)
{
    auto enc = tensor_map_encoder();
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

// rows x 64 bf16 (128-byte rows), box = 64 rows, 128-byte swizzle
bool make_rows_map(CUtensorMap *map, const void *base, int64_t rows)
{
    auto enc = tensor_map_encoder();
    if (!enc || rows <= 0 || rows > 0x7fffffffLL) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(kN), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(kN * 2)};
    cuuint32_t box[2] = {kN, 64};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time driver dependency)
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
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

int g_chunked_inject_timeout = 0;  // test hook: set through rwkv_debug_inject_timeout

namespace {
int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

// A split call that updates its state in place (sT == s0) needs a copy of s0 in scratch.
bool split_state_copy(const Wkv6Args &a) { return a.s0 != nullptr && a.sT == a.s0; }

// Pieces per segment of the first pass: segments are halved (and halved again) while the
// pieces keep >= 4 chunks and every (b, h, piece) CTA of the first pass fits on the GPU at
// once, so that pass takes the time of a shorter piece.
int64_t pieces_per_segment(int64_t bh, int64_t G, int64_t seg_chunks)
{
    if (G <= 1) return 1;
    const int64_t slots = static_cast<int64_t>(wkv6_chunk_state_ctas_per_sm()) * sm_count();
    int64_t m = 1;
    while (seg_chunks % (2 * m) == 0 && seg_chunks / (2 * m) >= 4 && bh * (G - 1) * 2 * m <= slots) m *= 2;
    return m;
}

// Kernel attributes (shared memory size, carveout), set once per device.
cudaError_t configure_kernel()
{
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return cudaSuccess;
    for (auto kern : {wkv6_chunked_kernel<false, false>, wkv6_chunked_kernel<true, false>,
                      wkv6_chunked_kernel<false, true>, wkv6_chunked_kernel<true, true>}) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    done[dev] = true;
    return cudaSuccess;
}

// Stream-ordered pool for the sequence-split scratch, one per device, owned by the library.
// It keeps up to kPoolKeepBytes reserved across synchronisations, so a call does not map
// fresh memory each time (the process-wide default pool hands freed memory back to the
// system at every synchronisation unless its release threshold is raised, and changing
// that pool's attributes would affect every other user of it).
constexpr uint64_t kPoolKeepBytes = 64ull << 20;

cudaError_t scratch_pool(cudaMemPool_t *out)
{
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t pool = nullptr;
        e = cudaMemPoolCreate(&pool, &props);
        if (e != cudaSuccess) return e;
        uint64_t keep = kPoolKeepBytes;
        e = cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
        if (e != cudaSuccess) {
            cudaMemPoolDestroy(pool);
            return e;
        }
        pools[dev] = pool;
    }
    *out = pools[dev];
    return cudaSuccess;
}
}  // namespace

cudaError_t wkv6_chunked_launch(const Wkv6Args &a, cudaStream_t s)
{
    if (!a.bf16) return wkv6_serial_launch(a, s);
    const int64_t bh = a.B * a.H;
    if (bh == 0) return cudaSuccess;
    if (bh > 0x7fffffffLL || a.T > 0x7fffffffLL - kC || a.B > 0x7fffffffLL || a.H > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const int64_t nchunks = (a.T + kC - 1) / kC;

    // Sequence split: with fewer (b, h) sequences than two per SM, cut each sequence into
    // segments of >= 4 chunks that run side by side; a first pass over pieces of the
    // segments gives every segment its exact incoming state.
    int64_t G = 1;
    if (a.segments == 0) {
        const int64_t slots = 2LL * sm_count();
        if (bh < slots) G = std::min<int64_t>(slots / bh, nchunks / 4);
    } else {
        G = std::min<int64_t>(a.segments, nchunks);
    }
    G = std::max<int64_t>(G, 1);
    const int64_t seg_chunks = (nchunks + G - 1) / G;
    G = (nchunks + seg_chunks - 1) / seg_chunks;
    if (G > 65535) return cudaErrorInvalidConfiguration;

    CUtensorMap mr, mk, mv, mw;
    if (!make_map(&mr, a.r, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mw, a.w, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = configure_kernel();
    if (e != cudaSuccess) return e;

    const int64_t m = pieces_per_segment(bh, G, seg_chunks);
    const int64_t nsub = (G - 1) * m;
    const int64_t seg_floats = bh * nsub * kSegStride;
    ChunkedParams prm{a.T, a.H, a.u, a.s0, static_cast<__nv_bfloat16 *>(a.y), a.sT, a.status,
                      g_chunked_inject_timeout ? 100u : 100000u, g_chunked_inject_timeout,
                      static_cast<int>(seg_chunks), nullptr, static_cast<int>(G), static_cast<int>(m),
                      static_cast<int>(nsub), seg_floats,
                      static_cast<const __nv_bfloat16 *>(a.g), a.ln_w, a.ln_b, a.eps};
    float *seg = nullptr;
    if (G > 1) {
        const int64_t copy_floats = split_state_copy(a) ? bh * kN * kN : 0;
        cudaMemPool_t pool = nullptr;
        e = scratch_pool(&pool);
        if (e != cudaSuccess) return e;
        e = cudaMallocFromPoolAsync(reinterpret_cast<void **>(&seg),
                                    static_cast<size_t>(seg_floats + copy_floats) * sizeof(float), pool, s);
        if (e != cudaSuccess) return e;
        float *s0copy = copy_floats ? seg + seg_floats : nullptr;
        const ChunkStateArgs sa{a.T, a.H, bh, static_cast<int>(seg_chunks / m), static_cast<int>(nsub), seg,
                                seg_floats, a.s0, s0copy, a.status, g_chunked_inject_timeout, a.omega};
        e = wkv6_chunk_state_launch(mk, mv, mw, sa, s);
        prm.seg = seg;
        if (s0copy) prm.s0 = s0copy;
    }
    if (e == cudaSuccess) {
        auto kern = prm.gate ? (a.omega ? wkv6_chunked_kernel<true, true> : wkv6_chunked_kernel<true, false>)
                             : (a.omega ? wkv6_chunked_kernel<false, true> : wkv6_chunked_kernel<false, false>);
        kern<<<dim3(static_cast<unsigned>(bh), static_cast<unsigned>(G)), kThreads, kSmemBytes, s>>>(mr, mk, mv,
                                                                                                   mw, prm);
        e = cudaGetLastError();
    }
    if (seg) {
        const cudaError_t f = cudaFreeAsync(seg, s);
        if (e == cudaSuccess) e = f;
    }
    return e;
}

}  // namespace wkv

// ------------------------------------------------------------------ fixed-scratch variant
// rwkv_wkv6_forward_bf16_noalloc keeps the sequence-split scratch in this fixed array
// instead of allocating it, for callers that may not allocate device memory at all.  Every
// GPU that loads the library holds the array until the process exits.  The kernels reach
// it through the address passed in their parameters.
namespace wkv {

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchBytes / sizeof(float)];

namespace {
std::mutex g_noalloc_mu;
float *g_noalloc_addr[64] = {nullptr};

// In host code g_noalloc_scratch only names a host-side stand-in; its device address is
// looked up once per device, with that device current.
cudaError_t noalloc_scratch_address(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_addr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_addr[dev];
    return cudaSuccess;
}
}  // namespace

cudaError_t wkv6_chunked_launch_noalloc(const Wkv6Args &a, int segments, size_t *scratch_needed,
                                        cudaStream_t s)
{
    *scratch_needed = 0;
    const int64_t bh = a.B * a.H;
    if (bh == 0) return cudaSuccess;
    if (bh > 0x7fffffffLL || a.T > 0x7fffffffLL - kC || a.B > 0x7fffffffLL || a.H > 0x7fffffffLL)
        return cudaErrorInvalidConfiguration;
    const int64_t nchunks = (a.T + kC - 1) / kC;
    const int64_t per_segment = static_cast<int64_t>(kSegStride) * sizeof(float) * bh;
    // an in-place split also keeps a copy of s0 in the array
    const int64_t copy_bytes = split_state_copy(a) ? bh * kN * kN * static_cast<int64_t>(sizeof(float)) : 0;
    const int64_t cap = static_cast<int64_t>(kNoAllocScratchBytes);
    int64_t G = 1;
    if (segments == 0) {  // as the allocating entry point, capped to what the array holds
        const int64_t slots = 2LL * sm_count();
        if (bh < slots) G = std::min<int64_t>(slots / bh, nchunks / 4);
        G = std::min<int64_t>(G, cap >= copy_bytes ? (cap - copy_bytes) / per_segment + 1 : 1);
    } else {
        G = std::min<int64_t>(segments, nchunks);
    }
    G = std::max<int64_t>(G, 1);
    const int64_t seg_chunks = (nchunks + G - 1) / G;
    G = (nchunks + seg_chunks - 1) / seg_chunks;
    if (G > 65535) return cudaErrorInvalidConfiguration;
    // first-pass pieces per segment, fewer if their entries do not fit in the array
    int64_t m = pieces_per_segment(bh, G, seg_chunks);
    while (m > 1 && (G - 1) * m * per_segment + copy_bytes > cap) m /= 2;
    const int64_t nsub = (G - 1) * m;
    *scratch_needed = G > 1 ? static_cast<size_t>(nsub * per_segment + copy_bytes) : 0;
    if (*scratch_needed > kNoAllocScratchBytes) return cudaErrorInvalidValue;

    float *seg = nullptr;
    if (G > 1) {
        cudaError_t e = noalloc_scratch_address(&seg);
        if (e != cudaSuccess) return e;
    }
    CUtensorMap mr, mk, mv, mw;
    if (!make_map(&mr, a.r, a.B, a.T, a.H) || !make_map(&mk, a.k, a.B, a.T, a.H) ||
        !make_map(&mv, a.v, a.B, a.T, a.H) || !make_map(&mw, a.w, a.B, a.T, a.H))
        return cudaErrorInvalidValue;
    cudaError_t e = configure_kernel();
    if (e != cudaSuccess) return e;
    const int64_t seg_floats = nsub * per_segment / static_cast<int64_t>(sizeof(float));
    ChunkedParams prm{a.T, a.H, a.u, a.s0, static_cast<__nv_bfloat16 *>(a.y), a.sT, a.status,
                      g_chunked_inject_timeout ? 100u : 100000u, g_chunked_inject_timeout,
                      static_cast<int>(seg_chunks), seg, static_cast<int>(G), static_cast<int>(m),
                      static_cast<int>(nsub), seg_floats,
                      static_cast<const __nv_bfloat16 *>(a.g), a.ln_w, a.ln_b, a.eps};
    if (G > 1) {
        // the first pass writes every scratch entry the full pass reads (the s0 copy of an
        // in-place call included): nothing in the array has to start at zero, and what an
        // earlier call left there is never read
        float *s0copy = copy_bytes ? seg + seg_floats : nullptr;
        const ChunkStateArgs sa{a.T, a.H, bh, static_cast<int>(seg_chunks / m), static_cast<int>(nsub), seg,
                                seg_floats, a.s0, s0copy, a.status, g_chunked_inject_timeout, false};
        e = wkv6_chunk_state_launch(mk, mv, mw, sa, s);
        if (e != cudaSuccess) return e;
        if (s0copy) prm.s0 = s0copy;
    }
    wkv6_chunked_kernel<false, false><<<dim3(static_cast<unsigned>(bh), static_cast<unsigned>(G)), kThreads,
                                        kSmemBytes, s>>>(
        mr, mk, mv, mw, prm);
    return cudaGetLastError();
}

}  // namespace wkv
