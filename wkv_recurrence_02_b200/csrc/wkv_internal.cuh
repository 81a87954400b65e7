// Internal declarations shared by the ABI layer and the kernel files of libwkv.so.
// Nothing here is part of the public ABI (include/rwkv_wkv.h is).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace wkv {

// Status codes written by kernels into the device status word (same values as rwkv_status).
constexpr int kStatusTimeout = -6;
constexpr int kStatusBounds = -9;

// Record the first device-side error; later errors keep the first one.
__device__ __forceinline__ void record_status(int *status, int code)
{
    if (status) atomicCAS(status, 0, code);
}

// Index checks of the debug build.  Compiled with WKV_DEBUG_BOUNDS, in_bounds() checks that the
// n elements from index i lie inside [0, limit), records RWKV_ERR_BOUNDS in the device status
// word when they do not, and returns the answer, so that the caller skips the access (nothing
// traps).  In ordinary builds it is the constant true and the checks compile away.
#ifdef WKV_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif
__device__ __forceinline__ bool in_bounds(int *status, int64_t i, int64_t n, int64_t limit)
{
    if (!kDebugBounds) return true;
    const bool ok = i >= 0 && n >= 0 && i + n <= limit;
    if (!ok) record_status(status, kStatusBounds);
    return ok;
}
// A TMA tile coordinate pair for an innermost coordinate x of element size es: x must start on
// a 16-byte boundary and inside the tensor, and the outer coordinate inside its extent.
__device__ __forceinline__ bool tma_coord_ok(int *status, int64_t x, int es, int64_t xdim, int64_t y, int64_t ydim)
{
    if (!kDebugBounds) return true;
    const bool ok = x >= 0 && x < xdim && (x * es) % 16 == 0 && y >= 0 && y < ydim;
    if (!ok) record_status(status, kStatusBounds);
    return ok;
}

struct Wkv4Args {
    int64_t B, T, C;
    const float *w, *u;     // [C]
    const void *k, *v;      // [B,T,C] fp32 or bf16
    const float *s0;        // [B,3,C] or null
    void *y;                // [B,T,C]
    float *sT;              // [B,3,C] or null
    bool bf16;
    int *status;
};

struct Wkv6Args {
    int64_t B, T, H, N;
    const void *r, *k, *v, *w;  // [B,T,H,N] fp32 or bf16
    const float *u;             // [H,N]
    const float *s0;            // [B,H,N,N] or null
    void *y;                    // [B,T,H,N]
    float *sT;                  // [B,H,N,N] or null
    bool bf16;
    int *status;
    int segments;               // chunked kernel: 0 = choose the sequence split, n = at most n
    // fused output stage (bf16 only): y = SiLU(g) * (ln_w * (o - mean) / sqrt(var + eps) + ln_b)
    // per (b, t, h) when g is non-null
    const void *g = nullptr;    // [B,T,H,N] bf16
    const float *ln_w = nullptr, *ln_b = nullptr;  // [H,N]
    float eps = 0.f;
    // decay given by its logit: w holds omega_t and the kernels form w_t = exp(-exp(omega_t))
    bool omega = false;
};

// WKV-6 backward: gradients (fp32) of a loss with dL/dy = dy and dL/dsT = dsT (null = 0).
struct Wkv6BwdArgs {
    int64_t B, T, H, N;
    const void *r, *k, *v, *w;  // [B,T,H,N] fp32 or bf16; w holds omega_t when omega is set
    const float *u;             // [H,N]
    const float *s0;            // [B,H,N,N] or null
    const void *dy;             // [B,T,H,N], dtype of r
    const float *dsT;           // [B,H,N,N] or null
    float *dr, *dk, *dv, *dw;   // [B,T,H,N]; dw is domega when omega is set
    float *du;                  // [H,N]
    float *ds0;                 // [B,H,N,N] or null
    void *workspace;            // wkv6_backward_workspace_bytes(B, T, H) bytes, 16-byte aligned
    bool bf16, omega;
    bool chunked = false;       // bf16 only: the tensor-core chunked backward (else the fp32 walks)
    int *status = nullptr;      // device status word (bounded waits that ran out)
};

// Byte layout of the backward workspace, shared by both backward paths.  The region at
// offset 0 holds either the fp32 walks' state checkpoints (one every 8 tokens) or the
// chunked path's bf16 checkpoints (state before each 64-token chunk and after the last,
// state gradient after each chunk) and its per-chunk row-dot terms; the walks run after
// the chunked kernels have finished with it (they serve the sequences the chunked path
// leaves to them).
struct BwdLayout {
    int64_t nch;                       // 64-token chunks
    size_t sck, dsck, rowdot;          // chunked: checkpoints and row dots (inside region 0)
    size_t du_part, du_item, flags;    // walks' du per (b, h); chunked du per (b, h, chunk); flags
    size_t total;
};
BwdLayout wkv6_backward_layout(int64_t B, int64_t T, int64_t H);
cudaError_t wkv6_backward_tc_launch(const Wkv6BwdArgs &a, const BwdLayout &L, cudaStream_t s);
// The fp32 walks; with `only` non-null they serve only the (b, h) whose flag is set.
cudaError_t wkv6_backward_walks_launch(const Wkv6BwdArgs &a, const BwdLayout &L, const int *only,
                                       cudaStream_t s);

size_t wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H);
cudaError_t wkv6_backward_launch(const Wkv6BwdArgs &a, cudaStream_t s);

// cuTensorMapEncodeTiled from the driver (null if unavailable).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// TMA tensor maps with the 128-byte swizzle, for bf16 tiles of 64 rows x 64 channels:
//   make_map:      a [B, T, H, 64] tensor, box = 64 tokens of one (b, h);
//   make_rows_map: a [rows, 64] array, box = 64 consecutive rows.
bool make_map(CUtensorMap *map, const void *base, int64_t B, int64_t T, int64_t H);
bool make_rows_map(CUtensorMap *map, const void *base, int64_t rows);

// Each launcher returns the cudaError_t of its launch(es).
cudaError_t wkv4_launch(const Wkv4Args &a, cudaStream_t s);
cudaError_t wkv6_serial_launch(const Wkv6Args &a, cudaStream_t s);
cudaError_t wkv6_decode_launch(const Wkv6Args &a, cudaStream_t s);
cudaError_t wkv6_chunked_launch(const Wkv6Args &a, cudaStream_t s);

// First pass of a split chunked prefill: for every (b, h) and every piece of sub_chunks
// 64-token chunks (pieces 0 .. nsub-1 of the sequence), the state the piece ends in when it
// starts from zero and the product of its decays, written to seg[bh][piece] as 64 x 64
// floats then 64 floats.  With s0copy set, the CTAs of piece 0 also copy s0 there (an
// in-place split call reads its initial state from the copy).  Maps as from make_map over k,
// v and w (w holding omega_t when omega is set).
struct ChunkStateArgs {
    int64_t T, H, bh;
    int sub_chunks, nsub;
    float *seg;
    int64_t seg_cap;          // floats behind seg
    const float *s0;
    float *s0copy;
    int *status;
    int inject_timeout;
    bool omega;
};
cudaError_t wkv6_chunk_state_launch(const CUtensorMap &mk, const CUtensorMap &mv, const CUtensorMap &mw,
                                    const ChunkStateArgs &a, cudaStream_t s);
// CTAs of the first-pass kernel that fit on one SM.
int wkv6_chunk_state_ctas_per_sm();

// The chunked kernel with its sequence-split scratch in a fixed device array (no
// allocation).  Returns cudaErrorInvalidValue with *scratch_needed > capacity when the
// requested split does not fit.
constexpr size_t kNoAllocScratchBytes = 4u << 20;
cudaError_t wkv6_chunked_launch_noalloc(const Wkv6Args &a, int segments, size_t *scratch_needed,
                                        cudaStream_t s);

// Test hook: when nonzero, chunked launches first wait on a barrier that is never
// signalled (short bound) so the timeout path runs; set via rwkv_debug_inject_timeout.
extern int g_chunked_inject_timeout;

}  // namespace wkv
