// rwkv_abi.cu -- the extern "C" boundary of libwkv.so (declared in include/rwkv_wkv.h).
//
// Host-side argument validation (before any CUDA call), kernel selection, the
// thread-local stream and the device status word.  Every step of the recurrences
// runs in the CUDA kernels of the other files; there is no CPU fallback.
#include "rwkv_wkv.h"
#include "wkv_internal.cuh"

#include <mutex>
#include <stdio.h>
#include <string.h>

namespace {

thread_local cudaStream_t tl_stream = nullptr;
thread_local int tl_wkv6_algo = RWKV_WKV6_AUTO;
thread_local int tl_wkv6_segments = 0;
thread_local char tl_err[256] = "";

// The library's only device memory: one status word per device, allocated statically.
__device__ int g_device_status = 0;

constexpr int kMaxDevices = 64;
std::mutex g_status_mu;
int *g_status_ptr[kMaxDevices] = {nullptr};

int fail(int code, const char *fmt, const char *detail = "")
{
    snprintf(tl_err, sizeof(tl_err), fmt, detail);
    return code;
}

int cuda_fail(cudaError_t e, const char *where)
{
    snprintf(tl_err, sizeof(tl_err), "%s: %s", where, cudaGetErrorString(e));
    return RWKV_ERR_CUDA;
}

// Device address of the status word on the current device (looked up once per device).
int status_word(int **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(RWKV_ERR_CUDA, "device index out of range%s");
    std::lock_guard<std::mutex> lock(g_status_mu);
    if (!g_status_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_device_status);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
        g_status_ptr[dev] = static_cast<int *>(p);
    }
    *out = g_status_ptr[dev];
    return RWKV_OK;
}

// ---- validation helpers -----------------------------------------------------------

bool mul_ok(int64_t a, int64_t b, int64_t *out)
{
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / 4 / a) return false;  // keep byte counts representable
    *out = a * b;
    return true;
}

struct Span {
    const void *p;
    int64_t bytes;
};

bool overlap(Span a, Span b)
{
    if (!a.p || !b.p || a.bytes <= 0 || b.bytes <= 0) return false;
    uintptr_t a0 = (uintptr_t)a.p, a1 = a0 + (uintptr_t)a.bytes;
    uintptr_t b0 = (uintptr_t)b.p, b1 = b0 + (uintptr_t)b.bytes;
    return a0 < b1 && b0 < a1;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// ---- WKV-4 -------------------------------------------------------------------------

int wkv4_entry(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
               const void *k, const void *v, const float *s0, void *y, float *sT,
               bool bf16, bool with_state)
{
    tl_err[0] = 0;
    if (B < 0 || T < 0 || C < 0) return fail(RWKV_ERR_SHAPE, "negative size%s");
    int64_t BT, n, ns;
    if (!mul_ok(B, T, &BT) || !mul_ok(BT, C, &n) || !mul_ok(B * 3, C, &ns))
        return fail(RWKV_ERR_SHAPE, "size product overflows%s");
    const int64_t esz = bf16 ? 2 : 4;
    const bool want_state = with_state && sT != nullptr;
    if (n == 0 && !(want_state && ns > 0)) return RWKV_OK;
    if (n > 0 && (!k || !v || !y)) return fail(RWKV_ERR_NULL, "k, v and y must be non-null%s");
    if (C > 0 && B > 0 && (!w || !u)) return fail(RWKV_ERR_NULL, "w and u must be non-null%s");
    const void *ptrs[] = {w, u, k, v, y, s0, sT};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(RWKV_ERR_ALIGN, "tensor pointers must be 16-byte aligned%s");
    Span sy{y, n * esz}, sk{k, n * esz}, sv{v, n * esz}, sw{w, C * 4}, su{u, C * 4};
    Span ss0{s0, with_state ? ns * 4 : 0}, ssT{sT, with_state ? ns * 4 : 0};
    if (overlap(sy, sk) || overlap(sy, sv) || overlap(sy, sw) || overlap(sy, su) ||
        overlap(sy, ss0) || overlap(sy, ssT))
        return fail(RWKV_ERR_ALIAS, "y overlaps another tensor%s");
    if (with_state && sT) {
        if (overlap(ssT, sk) || overlap(ssT, sv) || overlap(ssT, sw) || overlap(ssT, su))
            return fail(RWKV_ERR_ALIAS, "sT overlaps an input%s");
        if (s0 && s0 != sT && overlap(ssT, ss0))
            return fail(RWKV_ERR_ALIAS, "sT partially overlaps s0%s");
    }
    int *status = nullptr;
    int rc = status_word(&status);
    if (rc) return rc;
    wkv::Wkv4Args a{B, T, C, w, u, k, v, with_state ? s0 : nullptr, y,
                    with_state ? sT : nullptr, bf16, status};
    cudaError_t e = wkv::wkv4_launch(a, tl_stream);
    if (e != cudaSuccess) return cuda_fail(e, "wkv4 launch");
    return RWKV_OK;
}

// ---- WKV-6 -------------------------------------------------------------------------

int wkv6_entry(int64_t B, int64_t T, int64_t H, int64_t N, const void *r, const void *k,
               const void *v, const void *w, const float *u, const float *s0, void *y,
               float *sT, bool bf16, const void *g = nullptr, const float *ln_w = nullptr,
               const float *ln_b = nullptr, float eps = 0.f, bool gated = false, bool omega = false)
{
    tl_err[0] = 0;
    if (B < 0 || T < 0 || H < 0 || N < 0) return fail(RWKV_ERR_SHAPE, "negative size%s");
    int64_t BT, BTH, n, BH, ns;
    if (!mul_ok(B, T, &BT) || !mul_ok(BT, H, &BTH) || !mul_ok(BTH, N, &n) ||
        !mul_ok(B, H, &BH) || !mul_ok(BH, N * N, &ns))
        return fail(RWKV_ERR_SHAPE, "size product overflows%s");
    if (n == 0 && !(sT && ns > 0)) return RWKV_OK;
    if (N != 64) return fail(RWKV_ERR_UNSUPPORTED, "head size N must be 64%s");
    const int64_t esz = bf16 ? 2 : 4;
    if (n > 0 && (!r || !k || !v || !w || !y))
        return fail(RWKV_ERR_NULL, "r, k, v, w and y must be non-null%s");
    if (BH > 0 && !u) return fail(RWKV_ERR_NULL, "u must be non-null%s");
    if (gated) {
        if (n > 0 && !g) return fail(RWKV_ERR_NULL, "g must be non-null%s");
        if (H * N > 0 && (!ln_w || !ln_b)) return fail(RWKV_ERR_NULL, "ln_w and ln_b must be non-null%s");
        if (!(eps >= 0.f) || eps > 3.0e38f) return fail(RWKV_ERR_ARG, "eps must be finite and >= 0%s");
    }
    const void *ptrs[] = {r, k, v, w, u, s0, y, sT, g, ln_w, ln_b};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(RWKV_ERR_ALIGN, "tensor pointers must be 16-byte aligned%s");
    Span sy{y, n * esz}, sr{r, n * esz}, sk{k, n * esz}, sv{v, n * esz}, sw{w, n * esz};
    Span su{u, H * N * 4}, ss0{s0, ns * 4}, ssT{sT, ns * 4};
    Span sg{g, n * esz}, slw{ln_w, H * N * 4}, slb{ln_b, H * N * 4};
    const Span ins[] = {sr, sk, sv, sw, su, sg, slw, slb};
    for (const Span &s : ins)
        if (overlap(sy, s)) return fail(RWKV_ERR_ALIAS, "y overlaps an input%s");
    if (overlap(sy, ss0) || overlap(sy, ssT)) return fail(RWKV_ERR_ALIAS, "y overlaps a state%s");
    if (sT) {
        for (const Span &s : ins)
            if (overlap(ssT, s)) return fail(RWKV_ERR_ALIAS, "sT overlaps an input%s");
        if (s0 && s0 != sT && overlap(ssT, ss0))
            return fail(RWKV_ERR_ALIAS, "sT partially overlaps s0%s");
    }
    int *status = nullptr;
    int rc = status_word(&status);
    if (rc) return rc;
    if (T == 0) {  // nothing to scan: sT = s0, or the zero state
        if (!sT || sT == s0) return RWKV_OK;
        cudaError_t e = s0 ? cudaMemcpyAsync(sT, s0, ns * 4, cudaMemcpyDeviceToDevice, tl_stream)
                           : cudaMemsetAsync(sT, 0, ns * 4, tl_stream);
        return e == cudaSuccess ? RWKV_OK : cuda_fail(e, "T=0 state copy");
    }
    wkv::Wkv6Args a{B, T, H, N, r, k, v, w, u, s0, y, sT, bf16, status, tl_wkv6_segments};
    a.omega = omega;
    cudaError_t e;
    if (gated) {  // fused output stage: chunked for T > 1, decode for T == 1
        a.g = g;
        a.ln_w = ln_w;
        a.ln_b = ln_b;
        a.eps = eps;
        e = T > 1 ? wkv::wkv6_chunked_launch(a, tl_stream) : wkv::wkv6_decode_launch(a, tl_stream);
        if (e != cudaSuccess) return cuda_fail(e, "wkv6 gated launch");
        return RWKV_OK;
    }
    int algo = tl_wkv6_algo;
    if (algo == RWKV_WKV6_SERIAL || !bf16)
        e = (T == 1 && algo != RWKV_WKV6_SERIAL) ? wkv::wkv6_decode_launch(a, tl_stream)
                                                 : wkv::wkv6_serial_launch(a, tl_stream);
    else if (algo == RWKV_WKV6_CHUNKED || T > 1)
        e = wkv::wkv6_chunked_launch(a, tl_stream);
    else
        e = wkv::wkv6_decode_launch(a, tl_stream);
    if (e != cudaSuccess) return cuda_fail(e, "wkv6 launch");
    return RWKV_OK;
}

// ---- WKV-6 backward -----------------------------------------------------------------

int wkv6_bwd_sizes(int64_t B, int64_t T, int64_t H, int64_t N, int64_t *n, int64_t *ns, int64_t *hn)
{
    if (B < 0 || T < 0 || H < 0 || N < 0) return fail(RWKV_ERR_SHAPE, "negative size%s");
    int64_t BT, BTH, BH;
    if (!mul_ok(B, T, &BT) || !mul_ok(BT, H, &BTH) || !mul_ok(BTH, N, n) || !mul_ok(B, H, &BH) ||
        !mul_ok(BH, N * N, ns) || !mul_ok(H, N, hn))
        return fail(RWKV_ERR_SHAPE, "size product overflows%s");
    // workspace: per (b, h), a 64 x 64 fp32 checkpoint every 8 tokens and 64 floats
    const int64_t nblk = (T + 7) / 8;
    int64_t per_head, cells;
    if (!mul_ok(nblk, 4096, &per_head) || !mul_ok(BH, per_head + 64, &cells))
        return fail(RWKV_ERR_SHAPE, "workspace size overflows%s");
    return RWKV_OK;
}

int wkv6_bwd_entry(int64_t B, int64_t T, int64_t H, int64_t N, const void *r, const void *k, const void *v,
                   const void *w, const float *u, const float *s0, const void *dy, const float *dsT, float *dr,
                   float *dk, float *dv, float *dw, float *du, float *ds0, void *workspace, size_t wbytes,
                   bool bf16, bool omega)
{
    tl_err[0] = 0;
    int64_t n, ns, hn;
    int rc = wkv6_bwd_sizes(B, T, H, N, &n, &ns, &hn);
    if (rc) return rc;
    if (n == 0 && hn == 0 && !(ds0 && ns > 0)) return RWKV_OK;
    if (N != 64) return fail(RWKV_ERR_UNSUPPORTED, "head size N must be 64%s");
    if (n > 0 && (!r || !k || !v || !w || !dy))
        return fail(RWKV_ERR_NULL, "r, k, v, w (or omega) and dy must be non-null%s");
    if (n > 0 && (!dr || !dk || !dv || !dw)) return fail(RWKV_ERR_NULL, "dr, dk, dv and dw must be non-null%s");
    if (hn > 0 && (!u || !du)) return fail(RWKV_ERR_NULL, "u and du must be non-null%s");
    const size_t need = n > 0 ? wkv::wkv6_backward_workspace_bytes(B, T, H) : 0;
    if (need > 0 && !workspace) return fail(RWKV_ERR_NULL, "workspace must be non-null%s");
    if (wbytes < need) {
        snprintf(tl_err, sizeof(tl_err), "workspace holds %zu bytes; this call needs %zu", wbytes, need);
        return RWKV_ERR_ARG;
    }
    const void *ptrs[] = {r, k, v, w, u, s0, dy, dsT, dr, dk, dv, dw, du, ds0, workspace};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(RWKV_ERR_ALIGN, "tensor pointers must be 16-byte aligned%s");
    const int64_t esz = bf16 ? 2 : 4;
    const Span ins[] = {{r, n * esz}, {k, n * esz}, {v, n * esz}, {w, n * esz}, {u, hn * 4}, {s0, ns * 4},
                        {dy, n * esz}, {dsT, ns * 4}};
    const Span outs[] = {{dr, n * 4}, {dk, n * 4}, {dv, n * 4}, {dw, n * 4}, {du, hn * 4},
                         {ds0, ns * 4}, {workspace, static_cast<int64_t>(need)}};
    const int n_outs = sizeof(outs) / sizeof(outs[0]);
    for (int a = 0; a < n_outs; ++a) {
        for (const Span &x : ins) {
            // ds0 may be the very same array as dsT (in place); any other overlap is refused
            if (outs[a].p == ds0 && x.p == dsT && ds0 == dsT) continue;
            if (overlap(outs[a], x)) return fail(RWKV_ERR_ALIAS, "a gradient or the workspace overlaps an input%s");
        }
        for (int c = a + 1; c < n_outs; ++c)
            if (overlap(outs[a], outs[c])) return fail(RWKV_ERR_ALIAS, "two outputs overlap%s");
    }
    int *status = nullptr;
    rc = status_word(&status);
    if (rc) return rc;
    cudaError_t e = cudaSuccess;
    if (n == 0) {  // no token: du = 0, ds0 = dsT (or 0)
        if (hn > 0) e = cudaMemsetAsync(du, 0, hn * 4, tl_stream);
        if (e == cudaSuccess && ds0 && ns > 0 && ds0 != dsT)
            e = dsT ? cudaMemcpyAsync(ds0, dsT, ns * 4, cudaMemcpyDeviceToDevice, tl_stream)
                    : cudaMemsetAsync(ds0, 0, ns * 4, tl_stream);
        return e == cudaSuccess ? RWKV_OK : cuda_fail(e, "wkv6 backward without tokens");
    }
    wkv::Wkv6BwdArgs a{B, T, H, N, r, k, v, w, u, s0, dy, dsT, dr, dk, dv, dw, du, ds0, workspace, bf16, omega};
    a.chunked = bf16 && tl_wkv6_algo != RWKV_WKV6_SERIAL;
    a.status = status;
    e = wkv::wkv6_backward_launch(a, tl_stream);
    if (e != cudaSuccess) return cuda_fail(e, "wkv6 backward launch");
    return RWKV_OK;
}

// Allocation-free WKV-6 (bf16): same validation as wkv6_entry, chunked kernel only, the
// split's scratch in the library's fixed device array.
int wkv6_noalloc_entry(int64_t B, int64_t T, int64_t H, int64_t N, const void *r, const void *k,
                       const void *v, const void *w, const float *u, const float *s0, void *y,
                       float *sT, int segments)
{
    tl_err[0] = 0;
    if (segments < 0) return fail(RWKV_ERR_ARG, "segments must be >= 0%s");
    if (B < 0 || T < 0 || H < 0 || N < 0) return fail(RWKV_ERR_SHAPE, "negative size%s");
    int64_t BT, BTH, n, BH, ns;
    if (!mul_ok(B, T, &BT) || !mul_ok(BT, H, &BTH) || !mul_ok(BTH, N, &n) ||
        !mul_ok(B, H, &BH) || !mul_ok(BH, N * N, &ns))
        return fail(RWKV_ERR_SHAPE, "size product overflows%s");
    if (n == 0 && !(sT && ns > 0)) return RWKV_OK;
    if (N != 64) return fail(RWKV_ERR_UNSUPPORTED, "head size N must be 64%s");
    if (n > 0 && (!r || !k || !v || !w || !y))
        return fail(RWKV_ERR_NULL, "r, k, v, w and y must be non-null%s");
    if (BH > 0 && !u) return fail(RWKV_ERR_NULL, "u must be non-null%s");
    const void *ptrs[] = {r, k, v, w, u, s0, y, sT};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return fail(RWKV_ERR_ALIGN, "tensor pointers must be 16-byte aligned%s");
    Span sy{y, n * 2}, sr{r, n * 2}, sk{k, n * 2}, sv{v, n * 2}, sw{w, n * 2};
    Span su{u, H * N * 4}, ss0{s0, ns * 4}, ssT{sT, ns * 4};
    const Span ins[] = {sr, sk, sv, sw, su};
    for (const Span &s : ins)
        if (overlap(sy, s)) return fail(RWKV_ERR_ALIAS, "y overlaps an input%s");
    if (overlap(sy, ss0) || overlap(sy, ssT)) return fail(RWKV_ERR_ALIAS, "y overlaps a state%s");
    if (sT) {
        for (const Span &s : ins)
            if (overlap(ssT, s)) return fail(RWKV_ERR_ALIAS, "sT overlaps an input%s");
        if (s0 && s0 != sT && overlap(ssT, ss0))
            return fail(RWKV_ERR_ALIAS, "sT partially overlaps s0%s");
    }
    int *status = nullptr;
    int rc = status_word(&status);
    if (rc) return rc;
    if (T == 0) {
        if (!sT || sT == s0) return RWKV_OK;
        cudaError_t e = s0 ? cudaMemcpyAsync(sT, s0, ns * 4, cudaMemcpyDeviceToDevice, tl_stream)
                           : cudaMemsetAsync(sT, 0, ns * 4, tl_stream);
        return e == cudaSuccess ? RWKV_OK : cuda_fail(e, "T=0 state copy");
    }
    wkv::Wkv6Args a{B, T, H, N, r, k, v, w, u, s0, y, sT, true, status, segments};
    size_t need = 0;
    cudaError_t e = wkv::wkv6_chunked_launch_noalloc(a, segments, &need, tl_stream);
    if (e == cudaErrorInvalidValue && need > wkv::kNoAllocScratchBytes) {
        snprintf(tl_err, sizeof(tl_err),
                 "the requested sequence split needs %zu bytes of scratch; the fixed no-allocation "
                 "buffer holds %zu (use fewer segments)",
                 need, wkv::kNoAllocScratchBytes);
        return RWKV_ERR_SHAPE;
    }
    if (e != cudaSuccess) return cuda_fail(e, "wkv6 no-allocation launch");
    return RWKV_OK;
}

}  // namespace

extern "C" {

int rwkv_wkv4_forward(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                      const float *k, const float *v, float *y)
{
    return wkv4_entry(B, T, C, w, u, k, v, nullptr, y, nullptr, false, false);
}

int rwkv_wkv4_forward_bf16(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                           const uint16_t *k, const uint16_t *v, uint16_t *y)
{
    return wkv4_entry(B, T, C, w, u, k, v, nullptr, y, nullptr, true, false);
}

int rwkv_wkv4_forward_state(int64_t B, int64_t T, int64_t C, const float *w, const float *u,
                            const float *k, const float *v, const float *s0, float *y,
                            float *sT)
{
    return wkv4_entry(B, T, C, w, u, k, v, s0, y, sT, false, true);
}

int rwkv_wkv4_forward_state_bf16(int64_t B, int64_t T, int64_t C, const float *w,
                                 const float *u, const uint16_t *k, const uint16_t *v,
                                 const float *s0, uint16_t *y, float *sT)
{
    return wkv4_entry(B, T, C, w, u, k, v, s0, y, sT, true, true);
}

int rwkv_wkv6_forward(int64_t B, int64_t T, int64_t H, int64_t N, const float *r,
                      const float *k, const float *v, const float *w, const float *u,
                      const float *s0, float *y, float *sT)
{
    return wkv6_entry(B, T, H, N, r, k, v, w, u, s0, y, sT, false);
}

int rwkv_wkv6_forward_bf16(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r,
                           const uint16_t *k, const uint16_t *v, const uint16_t *w,
                           const float *u, const float *s0, uint16_t *y, float *sT)
{
    return wkv6_entry(B, T, H, N, r, k, v, w, u, s0, y, sT, true);
}

extern "C" int rwkv_wkv6_forward_gated_bf16(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r,
                                            const uint16_t *k, const uint16_t *v, const uint16_t *w,
                                            const float *u, const float *s0, const uint16_t *g,
                                            const float *ln_w, const float *ln_b, float eps, uint16_t *y,
                                            float *sT)
{
    return wkv6_entry(B, T, H, N, r, k, v, w, u, s0, y, sT, true, g, ln_w, ln_b, eps, true);
}

int rwkv_wkv6_forward_omega_bf16(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r,
                                 const uint16_t *k, const uint16_t *v, const uint16_t *omega,
                                 const float *u, const float *s0, const uint16_t *g, const float *ln_w,
                                 const float *ln_b, float eps, uint16_t *y, float *sT)
{
    // the output stage is fused when any of its three tensors is given; the gated checks then
    // reject a missing one
    const bool gated = g || ln_w || ln_b;
    return wkv6_entry(B, T, H, N, r, k, v, omega, u, s0, y, sT, true, g, ln_w, ln_b, gated ? eps : 0.f, gated,
                      true);
}

int rwkv_wkv6_forward_bf16_noalloc(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r,
                                   const uint16_t *k, const uint16_t *v, const uint16_t *w,
                                   const float *u, const float *s0, uint16_t *y, float *sT,
                                   int segments)
{
    return wkv6_noalloc_entry(B, T, H, N, r, k, v, w, u, s0, y, sT, segments);
}

int rwkv_wkv6_backward_workspace_bytes(int64_t B, int64_t T, int64_t H, int64_t N, size_t *bytes)
{
    tl_err[0] = 0;
    if (!bytes) return fail(RWKV_ERR_NULL, "bytes must be non-null%s");
    int64_t n, ns, hn;
    int rc = wkv6_bwd_sizes(B, T, H, N, &n, &ns, &hn);
    if (rc) return rc;
    *bytes = n > 0 ? wkv::wkv6_backward_workspace_bytes(B, T, H) : 0;
    return RWKV_OK;
}

int rwkv_wkv6_backward(int64_t B, int64_t T, int64_t H, int64_t N, const float *r, const float *k,
                       const float *v, const float *w, const float *u, const float *s0, const float *dy,
                       const float *dsT, float *dr, float *dk, float *dv, float *dw, float *du, float *ds0,
                       void *workspace, size_t workspace_bytes)
{
    return wkv6_bwd_entry(B, T, H, N, r, k, v, w, u, s0, dy, dsT, dr, dk, dv, dw, du, ds0, workspace,
                          workspace_bytes, false, false);
}

int rwkv_wkv6_backward_bf16(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r, const uint16_t *k,
                            const uint16_t *v, const uint16_t *w, const float *u, const float *s0,
                            const uint16_t *dy, const float *dsT, float *dr, float *dk, float *dv, float *dw,
                            float *du, float *ds0, void *workspace, size_t workspace_bytes)
{
    return wkv6_bwd_entry(B, T, H, N, r, k, v, w, u, s0, dy, dsT, dr, dk, dv, dw, du, ds0, workspace,
                          workspace_bytes, true, false);
}

int rwkv_wkv6_backward_omega_bf16(int64_t B, int64_t T, int64_t H, int64_t N, const uint16_t *r,
                                  const uint16_t *k, const uint16_t *v, const uint16_t *omega, const float *u,
                                  const float *s0, const uint16_t *dy, const float *dsT, float *dr, float *dk,
                                  float *dv, float *domega, float *du, float *ds0, void *workspace,
                                  size_t workspace_bytes)
{
    return wkv6_bwd_entry(B, T, H, N, r, k, v, omega, u, s0, dy, dsT, dr, dk, dv, domega, du, ds0, workspace,
                          workspace_bytes, true, true);
}

int rwkv_set_wkv6_algo(int algo)
{
    if (algo != RWKV_WKV6_AUTO && algo != RWKV_WKV6_SERIAL && algo != RWKV_WKV6_CHUNKED)
        return RWKV_ERR_ARG;
    tl_wkv6_algo = algo;
    return RWKV_OK;
}

int rwkv_get_wkv6_algo(void) { return tl_wkv6_algo; }

int rwkv_set_wkv6_segments(int segments)
{
    if (segments < 0) return RWKV_ERR_ARG;
    tl_wkv6_segments = segments;
    return RWKV_OK;
}

int rwkv_get_wkv6_segments(void) { return tl_wkv6_segments; }

int rwkv_debug_inject_timeout(int enable)
{
    int prev = wkv::g_chunked_inject_timeout;
    wkv::g_chunked_inject_timeout = enable ? 1 : 0;
    return prev;
}

void rwkv_set_stream(void *cuda_stream) { tl_stream = static_cast<cudaStream_t>(cuda_stream); }

void *rwkv_get_stream(void) { return tl_stream; }

int rwkv_get_device_status(void)
{
    int *p = nullptr;
    int rc = status_word(&p);
    if (rc) return rc;
    cudaError_t e = cudaStreamSynchronize(tl_stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int value = 0, zero = 0;
    e = cudaMemcpy(&value, p, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    e = cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "status clear");
    return value;
}

const char *rwkv_status_string(int status)
{
    switch (status) {
    case RWKV_OK: return "ok";
    case RWKV_ERR_NULL: return "required pointer is null";
    case RWKV_ERR_SHAPE: return "invalid size";
    case RWKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case RWKV_ERR_ALIAS: return "output overlaps an input";
    case RWKV_ERR_CUDA: return "CUDA error";
    case RWKV_ERR_TIMEOUT: return "device-side wait timed out";
    case RWKV_ERR_ALIGN: return "pointer not 16-byte aligned";
    case RWKV_ERR_ARG: return "invalid argument";
    case RWKV_ERR_BOUNDS: return "index check failed (debug build)";
    default: return "unknown status";
    }
}

const char *rwkv_last_error(void) { return tl_err; }

int rwkv_abi_version(void) { return RWKV_ABI_VERSION; }

int rwkv_debug_bounds(void) { return wkv::kDebugBounds ? 1 : 0; }

}  // extern "C"
