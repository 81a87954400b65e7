// Device helpers shared by the tensor-core kernels of libwkv.so (sm_100a): shared-memory
// tile addressing with the 128-byte swizzle, UMMA descriptors, tcgen05 MMA / TMEM access,
// mbarriers with bounded waits, TMA loads, and packed fp32 / bf16 arithmetic.  Internal:
// not part of the public ABI.
//
// Tiles are 64 rows x 128 bytes (64 bf16 per row) with the 128-byte swizzle, stored
// row-major.  For D[M x N] = A[M x K] B[K x N], an operand read along its rows is K-major
// and one read across its rows is MN-major.
#pragma once

#include "wkv_internal.cuh"

namespace wkv {
namespace tc {

constexpr int kTileRows = 64;
constexpr int kTile = kTileRows * 128;  // bytes of one bf16 64x64 tile

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

// The same product with A (M x K bf16, K-major) read from tensor memory at `a`: for M = 64,
// row m in lane (m % 16) + 32 (m / 16), as the accumulator's rows, two K elements per
// 32-bit column (the lower K index in the low half).
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t id, uint32_t acc)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
                 "r"(a), "l"(b), "r"(id), "r"(acc));
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

// One try_wait that may suspend the thread (no issue slots used) for up to ~20 us.
__device__ __forceinline__ bool bar_try_sleep(uint32_t bar, uint32_t phase)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred P;\n\tmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, P;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(phase), "r"(20000u)
                 : "memory");
    return ok != 0;
}

// Bounded wait; returns false if the limit (number of try_waits) ran out.
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t phase, uint32_t limit)
{
    for (uint32_t it = 0; it < limit; ++it)
        if (bar_try_sleep(bar, phase)) return true;
    return false;
}

// Bounded wait without suspending (lowest wake-up latency; used by the one issuing thread).
__device__ __forceinline__ bool bar_wait_spin(uint32_t bar, uint32_t phase, uint32_t limit)
{
    for (uint32_t it = 0; it < limit; ++it)
        if (bar_try(bar, phase)) return true;
    return false;
}

__device__ __forceinline__ void bar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Named barrier over `count` threads with an OR vote.
__device__ __forceinline__ int named_sync_or(int id, int count, int pred)
{
    int out;
    asm volatile("{\n\t.reg .pred P, Q;\n\tsetp.ne.s32 P, %1, 0;\n\t"
                 "barrier.red.or.pred Q, %2, %3, P;\n\tselp.s32 %0, 1, 0, Q;\n\t}"
                 : "=r"(out)
                 : "r"(pred), "r"(id), "r"(count)
                 : "memory");
    return out;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            int c2, int c3, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1, uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
                 : "memory");
}

// Untiled bulk copies (addresses 16-byte aligned, size a multiple of 16 bytes): global ->
// shared completing on an mbarrier, and shared -> global in the issuing thread's bulk group.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
}

// Tile store shared -> global (bulk group of the issuing thread); clipped at the tensor's bounds.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3, uint32_t src)
{
    asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until at most N of this thread's bulk groups still read shared memory (or are pending)
template <int N> __device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Prefetch a tile into L2 (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap *map, int c0, int c1, int c2, int c3)
{
    asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1), "r"(c2), "r"(c3)
                 : "memory");
}
__device__ __forceinline__ void tma_prefetch_2d(const CUtensorMap *map, int c0, int c1)
{
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// 16 TMEM lanes x 64 columns: threads 0-15 get columns [c, c+32), threads 16-31 get
// [c+32, c+64), each thread one lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
                 "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]),
                   "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
                   "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
                   "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 TMEM lanes x 16 columns in each half: threads 0-15 get columns [c, c+16), threads
// 16-31 get [c+32, c+48), each thread one lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 32;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 16 TMEM lanes x 32 columns of raw words: threads 0-15 store columns [c, c+16), threads
// 16-31 [c+16, c+32), each thread one lane; waits for the stores.
__device__ __forceinline__ void tmem_st16w(uint32_t taddr, const uint32_t (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
                 "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
                 "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32])
{
    asm volatile("tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, "
                 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
                 "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
                 "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
                 "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
                 "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
                 "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
                 "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
                 "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
                 "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
                 "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float tanh_approx(float x)
{
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
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

// ------------------------------------------------------------- packed fp32 pairs (f32x2)
// Two fp32 lanes in one 64-bit register; Blackwell executes mul/fma on both in one
// instruction.
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
__device__ __forceinline__ P2 mul2(P2 a, P2 b)
{
    P2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}
__device__ __forceinline__ P2 fma2(P2 a, P2 b, P2 c)
{
    P2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d.r) : "l"(a.r), "l"(b.r), "l"(c.r));
    return d;
}
__device__ __forceinline__ P2 add2(P2 a, P2 b)
{
    P2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d.r) : "l"(a.r), "l"(b.r));
    return d;
}
__device__ __forceinline__ P2 one2() { return pk(1.f, 1.f); }

// bf16 pair (low half = first channel) -> exact fp32 pair
__device__ __forceinline__ P2 unpack2(uint32_t x)
{
    P2 p;
    asm("{\n\t.reg .b32 l, h;\n\tshl.b32 l, %1, 16;\n\tand.b32 h, %1, 0xFFFF0000;\n\tmov.b64 %0, {l, h};\n\t}"
        : "=l"(p.r)
        : "r"(x));
    return p;
}
// fp32 pair -> bf16 pair, round to nearest even
__device__ __forceinline__ uint32_t pack2(P2 p)
{
    uint32_t d;
    asm("{\n\t.reg .f32 l, h;\n\tmov.b64 {l, h}, %1;\n\tcvt.rn.bf16x2.f32 %0, h, l;\n\t}" : "=r"(d) : "l"(p.r));
    return d;
}
__device__ __forceinline__ P2 rcp2(P2 x) { return pk(rcp_approx(lo(x)), rcp_approx(hi(x))); }
__device__ __forceinline__ P2 shfl_xor2(P2 x, int m)
{
    P2 y;
    y.r = __shfl_xor_sync(0xffffffffu, x.r, m);
    return y;
}
__device__ __forceinline__ P2 ld_p2(const float *p)
{
    const float2 f = *reinterpret_cast<const float2 *>(p);
    return pk(f.x, f.y);
}

// four channels of one token row: two packed pairs
struct Q4 {
    P2 a, b;  // channels (0, 1) and (2, 3)
};
__device__ __forceinline__ Q4 mul4(Q4 x, Q4 y) { return {mul2(x.a, y.a), mul2(x.b, y.b)}; }
__device__ __forceinline__ Q4 one4() { return {one2(), one2()}; }
__device__ __forceinline__ Q4 unpack4(uint2 x) { return {unpack2(x.x), unpack2(x.y)}; }
__device__ __forceinline__ uint2 pack4(Q4 x) { return make_uint2(pack2(x.a), pack2(x.b)); }
__device__ __forceinline__ Q4 shfl_xor4(Q4 x, int m) { return {shfl_xor2(x.a, m), shfl_xor2(x.b, m)}; }
__device__ __forceinline__ Q4 ld_q4(const float *p) { return {ld_p2(p), ld_p2(p + 2)}; }
__device__ __forceinline__ void st_q4(float *p, Q4 x)
{
    *reinterpret_cast<float4 *>(p) = make_float4(lo(x.a), hi(x.a), lo(x.b), hi(x.b));
}
__device__ __forceinline__ uint2 ld_u2(const unsigned char *tile, uint32_t off)
{
    return *reinterpret_cast<const uint2 *>(tile + off);
}
__device__ __forceinline__ void st_u2(unsigned char *tile, uint32_t off, uint2 x)
{
    *reinterpret_cast<uint2 *>(tile + off) = x;
}
// true if any of the four channels is below lim
__device__ __forceinline__ bool any_below(Q4 x, float lim)
{
    return (lo(x.a) < lim) | (hi(x.a) < lim) | (lo(x.b) < lim) | (hi(x.b) < lim);
}
// sum over the four channels of r * u * k
__device__ __forceinline__ float bonus4(Q4 r, Q4 u, Q4 k)
{
    const P2 acc = fma2(mul2(r.b, u.b), k.b, mul2(mul2(r.a, u.a), k.a));
    return lo(acc) + hi(acc);
}

// Decay from its logit (section 4.1.2: w = exp(-exp(omega))), as 2^(-2^(omega log2 e) log2 e)
// with two approximate base-2 exponentials.  omega = -inf gives 1, +inf gives 0; fp32 keeps a
// decay close to 1 apart from 1, which a bf16 w cannot (its largest value below 1 is 1 - 2^-8).
__device__ __forceinline__ float decay_of_logit(float om)
{
    constexpr float kLog2e = 1.4426950408889634f;
    return ex2_approx(-ex2_approx(om * kLog2e) * kLog2e);
}
__device__ __forceinline__ P2 decay2(P2 om) { return pk(decay_of_logit(lo(om)), decay_of_logit(hi(om))); }
__device__ __forceinline__ Q4 decay4(Q4 om) { return {decay2(om.a), decay2(om.b)}; }

}  // namespace tc
}  // namespace wkv
