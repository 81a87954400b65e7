// wkv6_chunk_state.cu -- end state of sequence pieces, the first pass of a split WKV-6
// prefill on B200 (tcgen05 + TMA + TMEM).
//
// Source: "RWKV-5/6 (Eagle and Finch)", section 4.1.2 (the state update S <- diag(w_t) S +
// k_t^T v_t, key channel i decayed by w_t[i]) and section 4.2.2 (per-token w_t).  A piece of
// the sequence that starts from a zero state ends in the state
//
//   S_piece = sum_i (k_i prod_{j>i} w_j)^T v_i   and carries the decay D_piece = prod_j w_j,
//
// so the state entering a later piece is a chain of S <- diag(D_piece) S + S_piece over the
// pieces before it, started from s0.  The chunked prefill splits long sequences into
// segments that run side by side; this kernel gives every segment its incoming state by
// computing (S_piece, D_piece) for pieces of half a segment (or a whole one), all at once.
//
// One CTA per (batch row, head, piece); it walks the piece in 64-token chunks.  Per chunk,
// on CUDA cores, Kh[i] = k_i prod_{j>i, j in chunk} w_j (every factor <= 1) and the chunk
// decay D; on the tensor core KV = Kh^T V (64 x 64, fp32 in TMEM, two buffers); and the
// running state, held in fp32 registers (thread = key channel row, 32 value columns), takes
// S <- diag(D) S + KV.  The product of a chunk does not wait for the state, so the tensor
// core never sits on the chunk-to-chunk chain.  k, v, w arrive by TMA into a 3-stage ring
// (24 KB per stage: three CTAs fit on one SM).
//
// Every mbarrier wait is bounded; on expiry the CTA records RWKV_ERR_TIMEOUT in the device
// status word, waits (bounded) for its own copies and products, frees its tensor memory and
// returns.
#include "tc_common.cuh"

#include <mutex>

namespace wkv {
namespace {
using namespace tc;

constexpr int kC = 64;                 // tokens per chunk
constexpr int kN = 64;                 // head size
constexpr int kThreads = 256;
constexpr int kStages = 3;
constexpr int SLOT_K = 0, SLOT_V = kTile, SLOT_W = 2 * kTile;
constexpr int kStageBytes = 3 * kTile;
// Once every prep warp has read its w rows, the W slot is free: the 16-token sub-block
// products (warp a: 64 floats at row 16a) and the chunk decay (64 floats at row 2) go there.
constexpr int W_HS = 0, W_ROW = 128, W_D = 2 * 128;
constexpr int OFF_BAR = kStages * kStageBytes;     // mbarriers (8 bytes each)
constexpr int OFF_MISC = OFF_BAR + 16 * 8;         // tmem base, abort flag, TMA count
constexpr int kSmemBytes = OFF_MISC + 64 + 1024;   // + alignment slack
constexpr uint32_t kTmemCols = 128;                // KV, two buffers of 64 columns
// Three CTAs per SM: shared memory (228 KB per SM, 1 KB of it reserved per CTA), registers
// (__launch_bounds__) and tensor memory (3 x 128 of 512 columns) all allow it.
constexpr int kCtasPerSm = 3;
static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "three CTAs per SM do not fit");
static_assert(kCtasPerSm * kTmemCols <= 512, "tensor memory of three CTAs exceeds an SM's");
constexpr int kSegStride = kN * kN + kN;           // S_piece, then D_piece

struct Params {
    int64_t T, H;
    int sub_chunks;      // chunks per piece
    int nsub;            // pieces per sequence computed here (grid y)
    float *seg;          // [B*H][nsub][kSegStride]
    int64_t seg_cap;     // floats behind seg (index checks of the debug build)
    const float *s0;     // in-place split: copied to s0copy by the CTAs of piece 0
    float *s0copy;
    int *status;
    uint32_t spin_limit;
    int inject_timeout;
};

__device__ __forceinline__ void issue_stage(unsigned char *sm, uint32_t bar_full0, const CUtensorMap *mk,
                                            const CUtensorMap *mv, const CUtensorMap *mw, int c, int cabs,
                                            int h, int b, int *status, int64_t T)
{
    const int s = c % kStages;
    if (!tma_coord_ok(status, 0, 2, kN, static_cast<int64_t>(cabs) * kC, T)) return;
    const uint32_t dst = smem_u32(sm + s * kStageBytes);
    const uint32_t bar = bar_full0 + 8 * s;
    bar_expect_tx(bar, kStageBytes);
    const int t0 = cabs * kC;
    tma_load_4d(dst + SLOT_K, mk, 0, h, t0, b, bar);
    tma_load_4d(dst + SLOT_V, mv, 0, h, t0, b, bar);
    tma_load_4d(dst + SLOT_W, mw, 0, h, t0, b, bar);
}

// Warp roles (256 threads):
//   warps 0-3  prep: warp a forms Kh for the 16-token sub-block a of each chunk (lane: half hf
//              of the sub-block, channel quad cq), after exchanging sub-block decay products;
//   warps 4-7  state: thread (q, lr, hi) holds row 16q + lr (a key channel) of the running
//              state, value columns 32 hi .. 32 hi + 31, in registers.  Lane 0 of warp 4 also
//              issues the first TMA copies and the products KV = Kh^T V; lane 0 of warp 5
//              refills a stage with chunk c + 3 once every state thread is done with chunk c.
// Hand-offs are mbarriers: stage full (TMA -> prep), prep done (prep -> product), KV full
// (tcgen05.commit -> state) and KV free (state -> product, and stage refill).
template <bool OMEGA>
__global__ void __launch_bounds__(kThreads, 3)
wkv6_chunk_state_kernel(const __grid_constant__ CUtensorMap map_k, const __grid_constant__ CUtensorMap map_v,
                        const __grid_constant__ CUtensorMap map_w, const Params p)
{
    extern __shared__ unsigned char smem_raw[];
    // aligned by an offset on the __shared__ array itself (not through an integer), so the
    // compiler keeps the shared state space: its accesses are shared loads and stores, which it
    // may reorder freely around global ones
    unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    volatile uint32_t *misc = reinterpret_cast<volatile uint32_t *>(sm + OFF_MISC);
    // misc: [0] TMEM base, [1] abort, [2] chunks whose TMA has been issued
    const uint32_t bar_full0 = smem_u32(&bars[0]);    // + 8 * stage
    const uint32_t bar_prep0 = smem_u32(&bars[3]);    // + 8 * stage
    const uint32_t bar_kvfull0 = smem_u32(&bars[6]);  // + 8 * buffer
    const uint32_t bar_kvfree0 = smem_u32(&bars[8]);  // + 8 * buffer
    const uint32_t bar_never = smem_u32(&bars[10]);
    const uint32_t bar_drain = smem_u32(&bars[11]);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t bh = blockIdx.x;
    const int64_t b = bh / p.H, h = bh % p.H;
    const int64_t T = p.T;
    const int g = blockIdx.y;              // piece of the sequence
    const int cb = g * p.sub_chunks;       // its first chunk
    const int nchunks_all = static_cast<int>((T + kC - 1) / kC);
    const int nchunks = max(0, min(p.sub_chunks, nchunks_all - cb));
    const uint32_t limit = p.spin_limit;
    const uint32_t spin_limit = p.spin_limit * 64u;
    const bool issuer = tid == 128;    // the products
    const bool refiller = tid == 160;  // the TMA refills after the first kStages chunks

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            bar_init(bar_full0 + 8 * s, 1);
            bar_init(bar_prep0 + 8 * s, 128);
        }
        for (int i = 0; i < 2; ++i) {
            bar_init(bar_kvfull0 + 8 * i, 1);
            bar_init(bar_kvfree0 + 8 * i, 128);
        }
        bar_init(bar_never, 1);
        bar_init(bar_drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        misc[1] = 0;
        misc[2] = 0;
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

    int issued = 0;
    if (issuer) {
        for (; issued < kStages && issued < nchunks; ++issued)
            issue_stage(sm, bar_full0, &map_k, &map_v, &map_w, issued, cb + issued, static_cast<int>(h),
                        static_cast<int>(b), p.status, T);
        misc[2] = issued;
    }
    if (refiller) issued = kStages < nchunks ? kStages : nchunks;
    int abort = 0;
    if (p.inject_timeout && tid == 0) abort = !bar_wait(bar_never, 0, limit);
    abort = __syncthreads_or(abort);
    if (abort) misc[1] = 1;

    if (warp < 4) {
        // ================================ prep ================================
        const int a = warp, hf = lane >> 4, cq = lane & 15;
        const int t0h = 16 * a + 8 * hf;
        const uint32_t cbyte = 8 * cq;
        for (int c = 0; c < nchunks && !abort; ++c) {
            const int s = c % kStages;
            unsigned char *st = sm + s * kStageBytes;
            const int64_t t0 = static_cast<int64_t>(cb + c) * kC;
            const int tv = static_cast<int>(T - t0 < kC ? T - t0 : kC);
            const int ok = bar_wait_spin(bar_full0 + 8 * s, (c / kStages) & 1, spin_limit);
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
            // this warp's own w rows are read: its sub-block product goes to its first two rows
            __syncwarp();
            float *hs = reinterpret_cast<float *>(st + SLOT_W + W_HS);
            if (hf == 0 && in_bounds(p.status, a * 16 * 32 + 4 * cq, 4, kTile / 4))
                st_q4(hs + a * 16 * 32 + 4 * cq, mul4(Gh, Go));
            if (named_sync_or(1, 128, !ok || misc[1])) {
                abort = 1;
                misc[1] = 1;
                break;
            }
            Q4 D = one4(), aft = one4();
#pragma unroll
            for (int be = 0; be < 4; ++be) {
                const Q4 gb = ld_q4(hs + be * 16 * 32 + 4 * cq);
                D = mul4(D, gb);
                aft = be > a ? mul4(aft, gb) : aft;
            }
            // Kh[t] = k_t prod_{j>t} w_j, in place
            Q4 run = hf ? aft : mul4(aft, Go);
#pragma unroll
            for (int m = 7; m >= 0; --m) {
                const int t = t0h + m;
                const uint32_t off = swz(t, cbyte);
                const uint2 kk = t < tv ? ld_u2(st + SLOT_K, off) : make_uint2(0u, 0u);
                st_u2(st + SLOT_K, off, pack4(mul4(unpack4(kk), run)));
                run = mul4(run, w[m]);
            }
            if (warp == 0 && hf == 0) st_q4(reinterpret_cast<float *>(st + SLOT_W + W_D) + 4 * cq, D);
            fence_async_smem();
            bar_arrive(bar_prep0 + 8 * s);
        }
    } else {
        // ================================ state ===============================
        const int q = warp - 4, hi = lane >> 4, lr = lane & 15;
        const uint32_t tlane = tbase + (static_cast<uint32_t>(32 * q) << 16);
        const int row = 16 * q + lr;
        const int colh = 32 * hi;
        const int64_t nstate = static_cast<int64_t>(gridDim.x) * kN * kN;
        if (p.s0copy && g == 0 && in_bounds(p.status, (bh * kN + row) * kN + colh, 32, nstate)) {
            const float4 *src = reinterpret_cast<const float4 *>(p.s0 + (bh * kN + row) * kN + colh);
            float4 *dst = reinterpret_cast<float4 *>(p.s0copy + (bh * kN + row) * kN + colh);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = src[i];
        }
        float S[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) S[i] = 0.f;
        float dprod = 1.f;
        for (int c = 0; c < nchunks && !abort; ++c) {
            const int s = c % kStages, bf = c & 1;
            unsigned char *st = sm + s * kStageBytes;
            int ok = 1;
            if (issuer) {
                // KV of chunk c into buffer bf, once its operands are formed and the buffer's
                // previous chunk (c - 2) has been read
                ok = bar_wait_spin(bar_prep0 + 8 * s, (c / kStages) & 1, spin_limit);
                if (ok && c >= 2) ok = bar_wait_spin(bar_kvfree0 + 8 * bf, ((c - 2) >> 1) & 1, spin_limit);
                if (ok) {
                    fence_after();
                    const uint32_t aK = smem_u32(st + SLOT_K), aV = smem_u32(st + SLOT_V);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks)
                        mma(tbase + 64 * bf, desc_mn(aK + 2048 * ks), desc_mn(aV + 2048 * ks), idesc(64, 1, 1), ks > 0);
                    mma_commit(bar_kvfull0 + 8 * bf);
                }
            }
            if (ok) ok = bar_wait_spin(bar_kvfull0 + 8 * bf, (c >> 1) & 1, spin_limit);
            // the warp decides together (its lanes meet here, then read TMEM warp-wide)
            if (__any_sync(0xffffffffu, !ok || misc[1])) {
                abort = 1;
                misc[1] = 1;
                break;
            }
            bar_try(bar_prep0 + 8 * s, (c / kStages) & 1);  // D of this chunk is visible
            fence_after();
            const float d = reinterpret_cast<const float *>(st + SLOT_W + W_D)[row];
            float kv[16];
            tmem_ld16(tlane + 64 * bf, kv);
#pragma unroll
            for (int n = 0; n < 16; ++n) S[n] = fmaf(d, S[n], kv[n]);
            tmem_ld16(tlane + 64 * bf + 16, kv);
#pragma unroll
            for (int n = 0; n < 16; ++n) S[16 + n] = fmaf(d, S[16 + n], kv[n]);
            fence_before();
            bar_arrive(bar_kvfree0 + 8 * bf);
            dprod *= d;
            // refill the stage of chunk c with chunk c + 3 as soon as every state thread has
            // read its D (the product of chunk c is then complete too); a thread other than the
            // issuer does it, so the next product is not held up
            if (refiller && issued < nchunks) {
                if (bar_wait_spin(bar_kvfree0 + 8 * bf, (c >> 1) & 1, spin_limit)) {
                    issue_stage(sm, bar_full0, &map_k, &map_v, &map_w, issued, cb + issued, static_cast<int>(h),
                                static_cast<int>(b), p.status, T);
                    ++issued;
                    misc[2] = issued;
                } else {
                    misc[1] = 1;  // the next vote of this warp ends the loop
                }
            }
        }
        if (!abort && in_bounds(p.status, (bh * p.nsub + g) * kSegStride, kSegStride, p.seg_cap)) {
            float *sg = p.seg + (bh * p.nsub + g) * kSegStride;
            float4 *dst = reinterpret_cast<float4 *>(sg + row * kN + colh);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(S[4 * i], S[4 * i + 1], S[4 * i + 2], S[4 * i + 3]);
            if (hi == 0) sg[kN * kN + row] = dprod;
        }
    }

    // ---- drain after an abort, then release tensor memory
    fence_before();
    abort = __syncthreads_or(abort | misc[1]);
    fence_after();
    if (abort) {
        record_status(p.status, kStatusTimeout);
        if (issuer) {
            mma_commit(bar_drain);
            const int n = misc[2];
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

cudaError_t configure_state_kernel()
{
    static std::mutex mu;
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (done[dev]) return cudaSuccess;
    for (auto kern : {wkv6_chunk_state_kernel<false>, wkv6_chunk_state_kernel<true>}) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    done[dev] = true;
    return cudaSuccess;
}
}  // namespace

int wkv6_chunk_state_ctas_per_sm() { return kCtasPerSm; }

cudaError_t wkv6_chunk_state_launch(const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mw,
                                    const ChunkStateArgs &a, cudaStream_t s)
{
    if (a.bh <= 0 || a.nsub <= 0) return cudaSuccess;
    if (a.bh > 0x7fffffffLL || a.nsub > 65535) return cudaErrorInvalidConfiguration;
    cudaError_t e = configure_state_kernel();
    if (e != cudaSuccess) return e;
    Params prm{a.T, a.H, a.sub_chunks, a.nsub, a.seg, a.seg_cap, a.s0, a.s0copy, a.status,
               a.inject_timeout ? 100u : 100000u, a.inject_timeout};
    auto kern = a.omega ? wkv6_chunk_state_kernel<true> : wkv6_chunk_state_kernel<false>;
    kern<<<dim3(static_cast<unsigned>(a.bh), static_cast<unsigned>(a.nsub)), kThreads, kSmemBytes, s>>>(mk, mv, mw,
                                                                                                        prm);
    return cudaGetLastError();
}

}  // namespace wkv
