// Thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers, TMA tiled loads, the tensor memory (TMEM) allocator, tcgen05
// MMAs with their shared-memory matrix descriptors, and TMEM loads/stores.
// Every wait here is bounded by %globaltimer: a wait that runs out sets the
// CTA's abort word and the device error word and returns false, so a broken
// protocol ends the kernel instead of hanging the GPU.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace ditk {

constexpr int kErrTimeout = 5;
// A single wait longer than this is treated as a broken protocol.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;  // 1 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed.  Bounded:
// gives up (returning false) when `abort` is set by another thread or when the
// wait has lasted kWaitLimitNs, in which case it sets `abort` and the device
// error word `err` itself.  Every lane of a warp that calls it must call it.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) { ok = true; break; }
            if ((it & 15u) == 0) {
                if (*abort) break;
                if (globaltimer() - t0 > kWaitLimitNs) {
                    *abort = 1;
                    atomicExch(err, kErrTimeout);
                    break;
                }
            }
        }
    }
    // Warp-uniform outcome: a lane that gave up makes the whole warp give up,
    // so warp-collective instructions after the wait stay converged.
    return __all_sync(0xffffffffu, ok);
}

// The same wait, polling 16 times between the checks of the abort word and
// the clock instead of keeping a poll counter: fewer instructions per poll on
// the SMSPs the waiting warps share with busy ones.  The bf16 attention kernel
// measured 2% faster with it; the 8-bit kernel measured 2% slower, so it keeps
// mbar_wait.
__device__ __forceinline__ bool mbar_wait_lean(uint64_t* bar, uint32_t parity, volatile int* abort, int* err) {
    bool ok = mbar_try_wait(bar, parity);
    if (!ok) {
        const uint64_t t0 = globaltimer();
        for (;;) {
            bool got = false;
#pragma unroll
            for (int u = 0; u < 16; ++u) {
                if (mbar_try_wait(bar, parity)) {
                    got = true;
                    break;
                }
            }
            if (got) {
                ok = true;
                break;
            }
            if (*abort) break;
            if (globaltimer() - t0 > kWaitLimitNs) {
                *abort = 1;
                atomicExch(err, kErrTimeout);
                break;
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

// Drain wait used on the way out of an aborted kernel: ignores the abort word
// (the copy or MMA being waited for still lands) but stays bounded in time.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    }
    return true;
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 4-D tiled TMA load into this CTA's shared memory; completion
// is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------- TMEM
// Allocate `ncols` (power of two, >= 32) TMEM columns; whole warp executes.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive 32-bit TMEM columns of this thread's lane (32x32b shape:
// warp w of a warpgroup reads lanes 32w..32w+31, one lane per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
// Ties the registers written by an earlier tcgen05.ld to this point in program
// order, so no use of them is scheduled above the preceding tcgen05.wait::ld.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
#pragma unroll
    for (int i = 0; i < 32; i += 8)
        asm volatile("" : "+r"(r[i]), "+r"(r[i + 1]), "+r"(r[i + 2]), "+r"(r[i + 3]), "+r"(r[i + 4]),
                     "+r"(r[i + 5]), "+r"(r[i + 6]), "+r"(r[i + 7]));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// ---------------------------------------------------------------- tcgen05.mma
// Shared-memory matrix descriptor (tcgen05 "matrix descriptor" format):
//   bits  0-13 start address >> 4       bits 16-29 leading byte offset >> 4
//   bits 32-45 stride byte offset >> 4  bits 46-47 version (1 on sm_100)
//   bits 49-51 base offset (0: atoms aligned to their own size)
//   bits 61-63 layout: 2 = 128-byte swizzle (8 rows × 128 B atoms),
//                      4 = 64-byte swizzle (8 rows × 64 B atoms)
constexpr uint32_t kLayoutSw128 = 2;
constexpr uint32_t kLayoutSw64 = 4;
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return smem_desc(saddr, lbo_bytes, sbo_bytes, kLayoutSw128);
}

// Instruction descriptor for kind::f16 / kind::i8 / kind::f8f6f4 (dense):
//   bits 4-5 D format (1 = f32, 2 = s32)   bits 7-9 A format   bits 10-12 B format
//   bit 15 A major (0 = K)   bit 16 B major (1 = MN)   bits 17-22 N >> 3
//   bits 24-28 M >> 4
__host__ __device__ constexpr uint32_t make_idesc(uint32_t dfmt, uint32_t afmt, uint32_t bfmt, uint32_t a_mn,
                                                  uint32_t b_mn, uint32_t M, uint32_t N) {
    return (dfmt << 4) | (afmt << 7) | (bfmt << 10) | (a_mn << 15) | (b_mn << 16) | ((N >> 3) << 17) |
           ((M >> 4) << 24);
}

// Shared-memory descriptors are passed as (low word, high word).  The start
// address lives in bits 0-13 of the low word in 16-byte units, so a
// descriptor for the same layout `bytes` further on is lo + bytes/16 (shared
// memory ends below 2^18 bytes: no carry leaves the field).  Building every
// descriptor once and advancing only its low word keeps the issuing thread's
// per-MMA work to one add, so MMAs issue at the tensor core's rate.
struct SDesc {
    uint32_t lo, hi;
};
__device__ __forceinline__ SDesc sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout) {
    const uint64_t d = smem_desc(saddr, lbo_bytes, sbo_bytes, layout);
    return SDesc{static_cast<uint32_t>(d), static_cast<uint32_t>(d >> 32)};
}
__device__ __forceinline__ SDesc sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return sdesc(saddr, lbo_bytes, sbo_bytes, kLayoutSw128);
}
__device__ __forceinline__ SDesc sdesc_add(SDesc d, uint32_t bytes) { return SDesc{d.lo + (bytes >> 4), d.hi}; }

// MMA issue is warp-collective: every lane of the (converged) issuing warp
// executes these with warp-uniform operands, and elect.sync picks the one lane
// that issues the instruction.  The same lane (the lowest, all lanes being
// active) issues every MMA and every commit, so a commit covers all MMAs the
// warp issued before it.  Issuing this way keeps the operands on the uniform
// datapath; guarding a single-thread issue with `lane == 0` made each MMA issue
// take 80-110 cycles next to busy softmax warps instead of about 40-60.
//
// D[tmem] (+)= A[smem] · B[smem] (kind::f16 / kind::i8), split descriptors.
template <int KIND>  // 0: f16 (bf16 in, fp32 acc), 1: i8 (s8 in, s32 acc)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, SDesc a, SDesc b, uint32_t idesc, uint32_t accumulate) {
    if (KIND == 0)
        asm volatile(
            "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
            "r"(a.lo), "r"(a.hi), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p, e;\n\t.reg .b64 da, db;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "mov.b64 da, {%1, %2};\n\tmov.b64 db, {%3, %4};\n\t"
            "setp.ne.b32 p, %6, 0;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::i8 [%0], da, db, %5, p;\n\t}" ::"r"(d_tmem),
            "r"(a.lo), "r"(a.hi), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
            : "memory");
}
// D[tmem] (+)= A[tmem] · B[smem] (kind::f16 / kind::f8f6f4), split descriptor.
template <int KIND>  // 0: f16, 2: f8f6f4
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, SDesc b, uint32_t idesc,
                                       uint32_t accumulate) {
    if (KIND == 0)
        asm volatile(
            "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "mov.b64 db, {%2, %3};\n\t"
            "setp.ne.b32 p, %5, 0;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p, e;\n\t.reg .b64 db;\n\t"
            "elect.sync _|e, 0xffffffff;\n\t"
            "mov.b64 db, {%2, %3};\n\t"
            "setp.ne.b32 p, %5, 0;\n\t"
            "@e tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], db, %4, p;\n\t}" ::"r"(d_tmem),
            "r"(a_tmem), "r"(b.lo), "r"(b.hi), "r"(idesc), "r"(accumulate)
            : "memory");
}
// Arrive (once) on `bar` when every tcgen05 operation the issuing lane started
// so far has completed (warp-collective, like the MMAs).
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------- registers
// Warpgroup-wide register re-allocation (every warp of the warpgroup executes
// it).  The per-thread counts of all warpgroups must add up to at most the
// registers the CTA was launched with.
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- math
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// 2^x for a pair of floats on the FMA pipe instead of MUFU.  Cody–Waite
// split x = j + r with j = round(x) (adding 1.5·2^23 leaves j in the low
// mantissa bits) and |r| <= 1/2; 2^r from a cubic (relative-error minimax on
// [-1/2, 1/2], fitted for this library, max relative error 7.5e-5, far below
// bf16's 2^-9); then j is added to the exponent field.  x is clamped at -125
// so the result stays a normal float (2^-125 stands in for anything smaller).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 jf = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 r = __ffma2_rn(jf, make_float2(-1.f, -1.f), x);
    float2 p = __ffma2_rn(make_float2(0.0551716685f, 0.0551716685f), r, make_float2(0.2426111251f, 0.2426111251f));
    p = __ffma2_rn(p, r, make_float2(0.6932609677f, 0.6932609677f));
    p = __ffma2_rn(p, r, make_float2(0.9999280572f, 0.9999280572f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// The same with a quadratic for 2^r (relative-error minimax on [-1/2, 1/2],
// fitted for this library, max relative error 1.73e-3): one FFMA2 fewer per
// pair, for P stored as e4m3, whose own rounding step is 2^-4 relative.
__device__ __forceinline__ float2 exp2_poly2q(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.f, 12582912.f));
    const float2 jf = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));
    const float2 r = __ffma2_rn(jf, make_float2(-1.f, -1.f), x);
    float2 p = __ffma2_rn(make_float2(0.2384289674f, 0.2384289674f), r, make_float2(0.7034480172f, 0.7034480172f));
    p = __ffma2_rn(p, r, make_float2(1.0004431359f, 1.0004431359f));
    return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                       __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Two fp32 -> packed bf16x2 (round to nearest even); `lo` goes to bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace ditk
