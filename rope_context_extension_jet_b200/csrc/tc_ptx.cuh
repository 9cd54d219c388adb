// tc_ptx.cuh -- inline-PTX wrappers for the sm_100a tensor-core path:
// TMA tiled loads, tcgen05 (TMEM allocation, MMA, commit, loads/stores) and
// the UMMA shared-memory / instruction descriptors.
//
// Descriptor bit layouts follow the PTX ISA's tcgen05 "shared memory
// descriptor" and "instruction descriptor" tables (sm_100a).
#pragma once

#include <stdint.h>

#include "jl_ptx.cuh"

namespace jl {

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(void* dst, const void* tmap, int x, int y, int z,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const void* tmap)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---------------------------------------------------------------- TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// columns [col, col+32) of TMEM lane (lane_base + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
          "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
          "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
        "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
        "%30, %31, %32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- MMA
// Warpgroup register reallocation (all four warps of a warpgroup execute it).
template <int N> __device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N> __device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// Fast base-2 exponential (ex2.approx.ftz: ~2 ulp, flushes denormals; ex2(-inf) = 0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Three-input maximum (max.f32 with three sources, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Packed two-lane fp32 arithmetic (fma/add .f32x2, sm_100): both lanes in one
// instruction, round-to-nearest like the scalar forms.
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 mul2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b)
{
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ---------------------------------------------------------------- CTA pairs
// The cta_group::2 forms: one MMA spans the two CTAs of a cluster pair.  Rows
// [0, 128) of A and of D live in CTA 0 (its shared memory / TMEM), rows
// [128, 256) in CTA 1; B is split along N, the first N/2 columns from CTA 0's
// shared memory and the rest from CTA 1's, at the same offsets.  Every tcgen05
// instruction of a kernel that uses them carries cta_group::2.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Warp-collective MMA issue and commits: the whole (converged) warp executes
// them with warp-uniform operands and one lane, chosen by elect.sync, issues
// the instructions.  Keeping the issuing loop on a full warp lets the
// descriptors live in uniform registers; a single divergent thread pays a
// per-instruction detour to make its operands uniform.  Commits of the pair
// kernel:
__device__ __forceinline__ void umma_commit_pair_both_elect(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;\n\t}" ::"r"(
            smem_u32(bar)),
        "h"((unsigned short)0x3)
        : "memory");
}
__device__ __forceinline__ void umma_commit_pair_local_elect(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// A whole K = 128 reduction as eight pair MMAs from one elected lane, with
// the descriptors of steps 1..7 made by adding immediates to the start-address
// field of step 0's (descriptor units of 16 bytes; every address stays below
// 2^18 bytes, so the 14-bit field never carries).  Q K^T: A = a 128-row
// K-major tile of two 64-column atoms (step k at (k / 4) * 1024 + (k % 4) * 2
// units), B = a 64-row K-major tile of two atoms (step k at (k / 4) * 512 +
// (k % 4) * 2); the first step overwrites D unless `acc0`.
__device__ __forceinline__ void umma_pair_qk_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t acc0)
{
    const uint32_t alo = (uint32_t)a_desc, ahi = (uint32_t)(a_desc >> 32);
    const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);
#define JL_QK_STEP(AO, BO)                                                                     \
    "add.u32 al, %1, " #AO ";\n\tadd.u32 bl, %3, " #BO ";\n\t"                              \
    "mov.b64 da, {al, %2};\n\tmov.b64 db, {bl, %4};\n\t"                                    \
    "@e tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, t;\n\t"
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 al, bl;\n\t.reg .b64 da, db;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "setp.eq.b32 t, %6, %6;\n\t"
        "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], da, db, %5, p;\n\t"
        JL_QK_STEP(2, 2) JL_QK_STEP(4, 4) JL_QK_STEP(6, 6)
        JL_QK_STEP(1024, 512) JL_QK_STEP(1026, 514) JL_QK_STEP(1028, 516) JL_QK_STEP(1030, 518)
        "}" ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
#undef JL_QK_STEP
}

// P V over a 128-key tile as eight pair MMAs from one elected lane: A = P in
// tensor memory (step k at column a_tmem + 8 k), B = an MN-major V tile whose
// K = 16 slices lie 2048 bytes apart (128 descriptor units); the first step
// overwrites D unless `acc0`.
__device__ __forceinline__ void umma_pair_pv_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                  uint32_t acc0)
{
    const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);
#define JL_PV_STEP(AO, BO)                                                                     \
    "add.u32 ta, %1, " #AO ";\n\tadd.u32 bl, %2, " #BO ";\n\t"                              \
    "mov.b64 db, {bl, %3};\n\t"                                                              \
    "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [ta], db, %4, t;\n\t"
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 ta, bl;\n\t.reg .b64 db;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 t, %5, %5;\n\t"
        "mov.b64 db, {%2, %3};\n\t"
        "@e tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], db, %4, p;\n\t"
        JL_PV_STEP(8, 128) JL_PV_STEP(16, 256) JL_PV_STEP(24, 384) JL_PV_STEP(32, 512)
        JL_PV_STEP(40, 640) JL_PV_STEP(48, 768) JL_PV_STEP(56, 896)
        "}" ::"r"(d_tmem), "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
#undef JL_PV_STEP
}

// The one-CTA forms (cta_group::1): Q K^T with A and B both 128-row K-major
// tiles (atoms 1024 units apart; D = 64 has one atom, four steps) and P V as
// in umma_pair_pv_k128.
#define JL_MMA1 "@e tcgen05.mma.cta_group::1.kind::f16 "
__device__ __forceinline__ void umma_qk_k128(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc)
{
    const uint32_t alo = (uint32_t)a_desc, ahi = (uint32_t)(a_desc >> 32);
    const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);
#define JL_QK1_STEP(O)                                                                          \
    "add.u32 al, %1, " #O ";\n\tadd.u32 bl, %3, " #O ";\n\t"                                 \
    "mov.b64 da, {al, %2};\n\tmov.b64 db, {bl, %4};\n\t" JL_MMA1 "[%0], da, db, %5, t;\n\t"
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 al, bl;\n\t.reg .b64 da, db;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %5, %5;\n\t"
        "setp.eq.b32 t, %5, %5;\n\t"
        "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t" JL_MMA1 "[%0], da, db, %5, p;\n\t"
        JL_QK1_STEP(2) JL_QK1_STEP(4) JL_QK1_STEP(6)
        JL_QK1_STEP(1024) JL_QK1_STEP(1026) JL_QK1_STEP(1028) JL_QK1_STEP(1030)
        "}" ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc)
        : "memory");
}
__device__ __forceinline__ void umma_qk_k64(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc)
{
    const uint32_t alo = (uint32_t)a_desc, ahi = (uint32_t)(a_desc >> 32);
    const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 al, bl;\n\t.reg .b64 da, db;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %5, %5;\n\t"
        "setp.eq.b32 t, %5, %5;\n\t"
        "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t" JL_MMA1 "[%0], da, db, %5, p;\n\t"
        JL_QK1_STEP(2) JL_QK1_STEP(4) JL_QK1_STEP(6)
        "}" ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc)
        : "memory");
#undef JL_QK1_STEP
}
__device__ __forceinline__ void umma_pv_k128(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t acc0)
{
    const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);
#define JL_PV1_STEP(AO, BO)                                                                     \
    "add.u32 ta, %1, " #AO ";\n\tadd.u32 bl, %2, " #BO ";\n\t"                               \
    "mov.b64 db, {bl, %3};\n\t" JL_MMA1 "[%0], [ta], db, %4, t;\n\t"
    asm volatile(
        "{\n\t.reg .pred p, t, e;\n\t.reg .b32 ta, bl;\n\t.reg .b64 db;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "setp.ne.b32 p, %5, 0;\n\t"
        "setp.eq.b32 t, %5, %5;\n\t"
        "mov.b64 db, {%2, %3};\n\t" JL_MMA1 "[%0], [%1], db, %4, p;\n\t"
        JL_PV1_STEP(8, 128) JL_PV1_STEP(16, 256) JL_PV1_STEP(24, 384) JL_PV1_STEP(32, 512)
        JL_PV1_STEP(40, 640) JL_PV1_STEP(48, 768) JL_PV1_STEP(56, 896)
        "}" ::"r"(d_tmem), "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)
        : "memory");
#undef JL_PV1_STEP
}
#undef JL_MMA1

// Arrive on `bar` once every tcgen05 operation this warp's elected lanes
// issued so far completed (one-CTA kernels, warp-collective).
__device__ __forceinline__ void umma_commit_elect(uint64_t* bar)
{
    asm volatile(
        "{\n\t.reg .pred e;\n\t"
        "elect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// Half of a P V: the four pair (cta_group::2) or one-CTA MMAs over 64 keys,
// A = P in tensor memory (step k at a_tmem + 8 k), B = V slices 128 descriptor
// units apart; the first step overwrites D unless `acc0`.  The second half of a
// tile is the same call at a_tmem + 32 and b_desc + 512.
#define JL_PVH(CG)                                                                                          \
    {                                                                                                       \
        const uint32_t blo = (uint32_t)b_desc, bhi = (uint32_t)(b_desc >> 32);                              \
        asm volatile(                                                                                       \
            "{\n\t.reg .pred p, t, e;\n\t.reg .b32 ta, bl;\n\t.reg .b64 db;\n\t"                      \
            "elect.sync _|e, 0xffffffff;\n\t"                                                               \
            "setp.ne.b32 p, %5, 0;\n\t"                                                                     \
            "setp.eq.b32 t, %5, %5;\n\t"                                                                    \
            "mov.b64 db, {%2, %3};\n\t"                                                                     \
            "@e tcgen05.mma.cta_group::" CG ".kind::f16 [%0], [%1], db, %4, p;\n\t"                       \
            "add.u32 ta, %1, 8;\n\tadd.u32 bl, %2, 128;\n\tmov.b64 db, {bl, %3};\n\t"                    \
            "@e tcgen05.mma.cta_group::" CG ".kind::f16 [%0], [ta], db, %4, t;\n\t"                       \
            "add.u32 ta, %1, 16;\n\tadd.u32 bl, %2, 256;\n\tmov.b64 db, {bl, %3};\n\t"                   \
            "@e tcgen05.mma.cta_group::" CG ".kind::f16 [%0], [ta], db, %4, t;\n\t"                       \
            "add.u32 ta, %1, 24;\n\tadd.u32 bl, %2, 384;\n\tmov.b64 db, {bl, %3};\n\t"                   \
            "@e tcgen05.mma.cta_group::" CG ".kind::f16 [%0], [ta], db, %4, t;\n\t"                       \
            "}" ::"r"(d_tmem), "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc0)                        \
            : "memory");                                                                                    \
    }
__device__ __forceinline__ void umma_pair_pv_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t acc0)
JL_PVH("2")
__device__ __forceinline__ void umma_pv_k64(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                            uint32_t acc0)
JL_PVH("1")
#undef JL_PVH

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
//   bits [0,14) start address >> 4; [16,30) leading byte offset >> 4;
//   [32,46) stride byte offset >> 4; [46,48) version = 1; [49,52) base offset = 0;
//   [52] LBO mode = 0; [61,64) layout = 2 (SWIZZLE_128B).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor for kind::f16 with fp16 A/B and fp32 accumulator
// (format fields 0 = f16); otherwise as idesc_bf16 below.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int b_mn_major)
{
    return (1u << 4) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 accumulator.
//   [4,6) D format = 1 (f32); [7,10) A format = 1 (bf16); [10,13) B format = 1;
//   [15] A major (0 = K); [16] B major (0 = K, 1 = MN); [17,23) N >> 3; [24,29) M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace jl
