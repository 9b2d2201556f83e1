// 8-bit softmax attention on sm_100a: S = Q8·K8ᵀ on tcgen05 kind::i8 (s32 in
// tensor memory), dequantised per (query block, key block), exp2 online
// softmax, and O += P·V either in FP8 e4m3 (kind::f8f6f4, P and V in e4m3) or
// in bf16 (kind::f16, P bf16, the caller's bf16 V).
//
// Method: "TMAP image-to-video inference acceleration", section on optimising
// operator details (8-bit SageAttention-style attention with per-block
// quantisation; the zero-scale guard).  The pre-pass (q8_prepass.cu) has
// written the INT8 codes of Q (per 128 tokens) and K (per 64 tokens, after
// the optional channel-mean subtraction), their scales, and for FP8 PV the
// per-channel e4m3 codes and scales of V.
//
// Structure as attn_bf16.cu (two 128-row query tiles per CTA, softmax
// warpgroups, one TMA warp, one MMA warp, S/P and O in tensor memory), with:
//   * logit of key c in log2 units t = acc·c_h, c_h = q_scale · k_scale(half h
//     of the key tile) · scale · log2 e.  |acc| <= 128·127² < 2^22, so
//     float(acc) = bits(acc + 0x4B400000) − 1.5·2^23 exactly, and the
//     subtraction folds into the exp argument's single FFMA;
//   * FP8 PV: P̃ = 2^(t − m + 6.5) is stored as e4m3.  The running max m
//     moves once a tile's max passes it by 2, so P̃ <= 2^8.5 < 448 and typical
//     weights stay in e4m3's normal range.  l sums the fp32 P̃, and the
//     epilogue multiplies O by v_scale[c] / l;
//   * bf16 PV: P = 2^(t − m), threshold 8, as in the bf16 kernel.
//
// Head dimension d = 128 or 64.  The 1-byte tiles (Q, K codes and e4m3 V)
// have d-byte rows: 128-byte swizzle at d = 128, 64-byte swizzle at d = 64;
// the bf16 V tile is d/64 panels of 64 elements with 128-byte swizzle.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "sm100_ptx.cuh"

namespace ditk {
namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kPanel = 128 * 128;  // 128 rows × 128 B swizzled panel (bf16 V)

template <bool FP8, int D>
struct Q8Cfg {
    static constexpr int kQTile = kBM * D;                 // int8
    static constexpr int kKTile = kBN * D;                 // int8
    static constexpr int kVTile = FP8 ? kBN * D : kBN * D * 2;
    static constexpr int kStages = FP8 ? 4 : 3;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = 2 * kQTile;
    static constexpr int kVOff = kKOff + kStages * kKTile;
    static constexpr int kBarOff = kVOff + kStages * kVTile;
    static constexpr int kNumBars = 1 + 4 * kStages + 6 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;
    // 1-byte tiles: rows of D bytes, swizzled over D bytes (8-row atoms).
    static constexpr uint32_t kLayout8 = D == 128 ? kLayoutSw128 : kLayoutSw64;
    static constexpr uint32_t kAtom8 = 8 * D;  // bytes per 8-row atom
    // Q8·K8ᵀ: s32 accumulate, signed int8 A/B, K-major.
    static constexpr uint32_t kIdescQK = make_idesc(2, 1, 1, 0, 0, 128, kBN);
    // P·V: fp32 accumulate; e4m3 × e4m3 (kind::f8f6f4) or bf16 × bf16, V MN-major.
    static constexpr uint32_t kIdescPV = FP8 ? make_idesc(1, 0, 0, 0, 1, 128, D) : make_idesc(1, 1, 1, 0, 1, 128, D);
    static constexpr float kShift = FP8 ? 6.5f : 0.0f;     // log2 of P's scale
    static constexpr float kThresh = FP8 ? 2.0f : 8.0f;    // rescale threshold (log2)
    // exp2 pairs (of 8) on the FMA pipe (tuned): FP8 P takes the quadratic
    // (exp2_poly2q, 3 pairs in 8), bf16 P the cubic (1 in 8).
    static constexpr int kEmuOf8 = FP8 ? 3 : 1;
};

struct Bars {
    uint64_t *q_full, *k_full, *k_empty, *v_full, *v_empty, *s_full, *p_full, *o_ready, *mma_done;
};

template <bool FP8, int D>
__device__ __forceinline__ Bars carve(uint8_t* base) {
    using C = Q8Cfg<FP8, D>;
    uint64_t* b = reinterpret_cast<uint64_t*>(base + C::kBarOff);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + C::kStages;
    r.v_full = r.k_empty + C::kStages;
    r.v_empty = r.v_full + C::kStages;
    r.s_full = r.v_empty + C::kStages;
    r.p_full = r.s_full + 2;
    r.o_ready = r.p_full + 2;
    r.mma_done = r.o_ready + 2;
    return r;
}

// Four fp32 -> four e4m3 in one word (round to nearest even, saturating);
// element 0 in bits 0-7.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint16_t lo, hi;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(lo) : "f"(b), "f"(a));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(hi) : "f"(d), "f"(c));
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

template <bool FP8, int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_q8_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                       const __grid_constant__ CUtensorMap tv, const float* __restrict__ q_scale,
                       const float* __restrict__ k_scale, const float* __restrict__ v_scale,
                       __nv_bfloat16* __restrict__ o, int64_t sb, int64_t sh, int64_t sn, int H, int N, int n_pairs,
                       float scale_log2, int* err) {
    using C = Q8Cfg<FP8, D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Bars bars = carve<FP8, D>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x % n_pairs;
    const int bh = blockIdx.x / n_pairs;
    const int b = bh / H;
    const int h = bh % H;
    const int q0 = pair * 2 * kBM;
    const int nkv = (N + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars.s_full[t], 1);
            mbar_init(&bars.p_full[t], kBM);
            mbar_init(&bars.o_ready[t], 1);
        }
        mbar_init(bars.mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t smem_base = smem_u32(smem);

    if (warp >= 8) {
        regs_dec<kOtherRegs>();
        if (warp == kLoadWarp) {
            // -------------------------------------------------------- TMA producer
            if (lane == 0) {
                tma_prefetch_desc(&tq);
                tma_prefetch_desc(&tk);
                tma_prefetch_desc(&tv);
                mbar_arrive_expect_tx(bars.q_full, 2 * C::kQTile);
                for (int t = 0; t < 2; ++t)
                    tma_load_4d(smem + C::kQOff + t * C::kQTile, &tq, bars.q_full, 0, q0 + t * kBM, h, b);
            }
            __syncwarp();
            int nk[C::kStages], nv[C::kStages];
#pragma unroll
            for (int s = 0; s < C::kStages; ++s) nk[s] = nv[s] = 0;
            for (int j = 0; j < nkv; ++j) {
                const int s = j % C::kStages;
                const uint32_t ph = (j / C::kStages) & 1;
                if (j >= C::kStages && !mbar_wait(&bars.k_empty[s], ph ^ 1, abort_flag, err)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars.k_full[s], C::kKTile);
                    tma_load_4d(smem + C::kKOff + s * C::kKTile, &tk, &bars.k_full[s], 0, j * kBN, h, b);
                }
                __syncwarp();
                ++nk[s];
                if (j >= C::kStages && !mbar_wait(&bars.v_empty[s], ph ^ 1, abort_flag, err)) break;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bars.v_full[s], C::kVTile);
                    if (FP8) {
                        tma_load_4d(smem + C::kVOff + s * C::kVTile, &tv, &bars.v_full[s], 0, j * kBN, h, b);
                    } else {
                        for (int hf = 0; hf < D / 64; ++hf)
                            tma_load_4d(smem + C::kVOff + s * C::kVTile + hf * kPanel, &tv, &bars.v_full[s], hf * 64,
                                        j * kBN, h, b);
                    }
                }
                __syncwarp();
                ++nv[s];
            }
            if (*abort_flag && lane == 0) {
                mbar_wait_drain(bars.q_full, 0);
                for (int s = 0; s < C::kStages; ++s) {
                    if (nk[s] > 0) mbar_wait_drain(&bars.k_full[s], (nk[s] - 1) & 1);
                    if (nv[s] > 0) mbar_wait_drain(&bars.v_full[s], (nv[s] - 1) & 1);
                }
            }
        } else if (warp == kMmaWarp) {
            // -------------------------------------------------------- MMA issuer
            // Descriptors are built once and advanced by byte offsets (SDesc).
            // K-major int8 operand: k-step kk = 32 bytes inside the D-byte
            // swizzled row (SBO = one 8-row atom).
            // V, MN-major: FP8 rows are one D-byte swizzled panel (k-step 32
            // keys, SBO = one 8-key atom); bf16 is D/64 panels of 64
            // elements, 16 KB apart (LBO), with 128-byte swizzle (k-step 16 keys).
            const SDesc dQ0 = sdesc(smem_base + C::kQOff, 16, C::kAtom8, C::kLayout8);
            const SDesc dQ1 = sdesc_add(dQ0, C::kQTile);
            const SDesc dK0 = sdesc(smem_base + C::kKOff, 16, C::kAtom8, C::kLayout8);
            const SDesc dV0 = FP8 ? sdesc(smem_base + C::kVOff, kPanel, C::kAtom8, C::kLayout8)
                                  : sdesc_sw128(smem_base + C::kVOff, kPanel, 1024);
            const uint32_t tS0 = tmem, tS1 = tmem + 128;
            const uint32_t tO0 = tmem + 256, tO1 = tmem + 256 + D;
            constexpr int kQKSteps = D / 32;
            constexpr int kPVSteps = FP8 ? kBN / 32 : kBN / 16;
            constexpr uint32_t kVStep = FP8 ? 32 * D : 16 * 128;
            auto issue_s = [&](uint32_t tS, SDesc dQ, SDesc dK) {
#pragma unroll
                for (int kk = 0; kk < kQKSteps; ++kk)
                    mma_ss<1>(tS, sdesc_add(dQ, kk * 32), sdesc_add(dK, kk * 32), C::kIdescQK, kk > 0);
            };
            auto issue_pv = [&](uint32_t tO, uint32_t tP, SDesc dV, bool acc) {
#pragma unroll
                for (int kk = 0; kk < kPVSteps; ++kk)
                    mma_ts<FP8 ? 2 : 0>(tO, tP + kk * 8, sdesc_add(dV, kk * kVStep), C::kIdescPV, acc || kk > 0);
            };
            bool ok = mbar_wait(bars.q_full, 0, abort_flag, err) && mbar_wait(&bars.k_full[0], 0, abort_flag, err);
            if (ok) {
                tc_fence_after();
                issue_s(tS0, dQ0, dK0);
                mma_commit(&bars.s_full[0]);
                issue_s(tS1, dQ1, dK0);
                mma_commit(&bars.s_full[1]);
                mma_commit(&bars.k_empty[0]);
                __syncwarp();
                for (int j = 0; j < nkv && ok; ++j) {
                    const int vs = j % C::kStages;
                    const SDesc dV = sdesc_add(dV0, vs * C::kVTile);
                    const bool more = j + 1 < nkv;
                    const int ks = (j + 1) % C::kStages;
                    const SDesc dK = sdesc_add(dK0, ks * C::kKTile);
                    ok = mbar_wait(&bars.v_full[vs], (j / C::kStages) & 1, abort_flag, err) &&
                         mbar_wait(&bars.p_full[0], j & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(tO0, tS0, dV, j > 0);
                    mma_commit(&bars.o_ready[0]);
                    __syncwarp();
                    if (more) {
                        ok = mbar_wait(&bars.k_full[ks], ((j + 1) / C::kStages) & 1, abort_flag, err);
                        if (!ok) break;
                        tc_fence_after();
                        issue_s(tS0, dQ0, dK);
                        mma_commit(&bars.s_full[0]);
                        __syncwarp();
                    }
                    ok = mbar_wait(&bars.p_full[1], j & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                    issue_pv(tO1, tS1, dV, j > 0);
                    mma_commit(&bars.o_ready[1]);
                    mma_commit(&bars.v_empty[vs]);
                    if (more) {
                        issue_s(tS1, dQ1, dK);
                        mma_commit(&bars.s_full[1]);
                        mma_commit(&bars.k_empty[ks]);
                    }
                    __syncwarp();
                }
            }
            mma_commit(bars.mma_done);
            if (lane == 0) mbar_wait_drain(bars.mma_done, 0);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        regs_inc<kSoftmaxRegs>();
        const int wg = warp >> 2;
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + wg * 128;
        const uint32_t tO = tmem + lane_off + 256 + wg * D;
        const int n_qblk = (N + 127) / 128, n_kblk = (N + 63) / 64;
        const int qtile = (q0 >> 7) + wg;
        // The second tile of the last pair can lie wholly past N: its rows are
        // padding, never stored; any finite scale serves.
        const float qs = qtile < n_qblk ? q_scale[static_cast<int64_t>(bh) * n_qblk + qtile] : 0.f;
        const float cq = qs * scale_log2;
        const float* ksc = k_scale + static_cast<int64_t>(bh) * n_kblk;
        constexpr float kBias = 12582912.0f;  // 1.5 · 2^23
        float m = -INFINITY;
        float l = 0.f;
        bool ok = true;
        float ks0 = ksc[0], ks1 = 1 < n_kblk ? ksc[1] : 0.f;
        for (int j = 0; j < nkv; ++j) {
            const float c0 = cq * ks0, c1 = cq * ks1;
            // next tile's key-block scales, loaded ahead
            if (j + 1 < nkv) {
                ks0 = ksc[2 * (j + 1)];
                ks1 = 2 * (j + 1) + 1 < n_kblk ? ksc[2 * (j + 1) + 1] : 0.f;
            }
            ok = mbar_wait(&bars.s_full[wg], j & 1, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, r[c]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 4; ++c) reg_fence32(r[c]);
            const int valid = N - j * kBN;  // keys of this tile below N
            const bool tail = valid < kBN;
            // Row max per key half, on the integers.
            int im0 = static_cast<int>(r[0][0]), im1 = static_cast<int>(r[2][0]);
            if (!tail) {
#pragma unroll
                for (int i = 1; i < 63; i += 2) {
                    im0 = __vimax3_s32(im0, static_cast<int>(r[i >> 5][i & 31]), static_cast<int>(r[(i + 1) >> 5][(i + 1) & 31]));
                    im1 = __vimax3_s32(im1, static_cast<int>(r[2 + (i >> 5)][i & 31]),
                                       static_cast<int>(r[2 + ((i + 1) >> 5)][(i + 1) & 31]));
                }
                im0 = max(im0, static_cast<int>(r[1][31]));
                im1 = max(im1, static_cast<int>(r[3][31]));
            } else {
                im0 = im1 = INT_MIN;
#pragma unroll
                for (int i = 0; i < 64; ++i) {
                    if (i < valid) im0 = max(im0, static_cast<int>(r[i >> 5][i & 31]));
                    if (64 + i < valid) im1 = max(im1, static_cast<int>(r[2 + (i >> 5)][i & 31]));
                }
            }
            float tmax = -INFINITY;
            if (im0 != INT_MIN) tmax = static_cast<float>(im0) * c0;
            if (im1 != INT_MIN) tmax = fmaxf(tmax, static_cast<float>(im1) * c1);
            const float m_new = fmaxf(m, tmax);
            if (j == 0) {
                m = m_new;
            } else {
                const bool need = m_new > m + C::kThresh;
                if (__any_sync(0xffffffffu, need)) {
                    ok = mbar_wait(&bars.o_ready[wg], (j - 1) & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                    const float alpha = need ? ex2_approx(m - m_new) : 1.0f;
                    const float2 alpha2 = make_float2(alpha, alpha);
                    uint32_t ro[32];
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        tmem_ld32(tO + c * 32, ro);
                        tmem_wait_ld();
                        reg_fence32(ro);
#pragma unroll
                        for (int i = 0; i < 32; i += 2) {
                            const float2 v = __fmul2_rn(
                                make_float2(__uint_as_float(ro[i]), __uint_as_float(ro[i + 1])), alpha2);
                            ro[i] = __float_as_uint(v.x);
                            ro[i + 1] = __float_as_uint(v.y);
                        }
                        tmem_st32(tO + c * 32, ro);
                    }
                    tmem_wait_st();
                    if (need) {
                        l *= alpha;
                        m = m_new;
                    }
                }
            }
            // exp argument: (acc + 1.5·2^23)·c_h − (1.5·2^23·c_h + m − shift)
            const float nb0 = -fmaf(kBias, c0, m - C::kShift);
            const float nb1 = -fmaf(kBias, c1, m - C::kShift);
            float2 ls[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
            float p[kBN];
#pragma unroll
            for (int i = 0; i < kBN; i += 2) {
                const float2 cc = i < 64 ? make_float2(c0, c0) : make_float2(c1, c1);
                const float2 nb = i < 64 ? make_float2(nb0, nb0) : make_float2(nb1, nb1);
                const float2 f = make_float2(__int_as_float(static_cast<int>(r[i >> 5][i & 31]) + 0x4B400000),
                                             __int_as_float(static_cast<int>(r[(i + 1) >> 5][(i + 1) & 31]) + 0x4B400000));
                const float2 t = __ffma2_rn(f, cc, nb);
                if (((i >> 1) & 7) < C::kEmuOf8) {
                    const float2 e = FP8 ? exp2_poly2q(t) : exp2_poly2(t);
                    p[i] = e.x;
                    p[i + 1] = e.y;
                } else {
                    p[i] = ex2_approx(t.x);
                    p[i + 1] = ex2_approx(t.y);
                }
            }
            if (tail) {
#pragma unroll
                for (int i = 0; i < kBN; ++i)
                    if (i >= valid) p[i] = 0.f;
            }
#pragma unroll
            for (int i = 0; i < kBN; i += 2) ls[(i >> 1) & 3] = __fadd2_rn(ls[(i >> 1) & 3], make_float2(p[i], p[i + 1]));
            if (FP8) {
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) pk[i] = e4m3x4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
                tmem_st32(tS, pk);
            } else {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t pk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(p[c * 64 + 2 * i], p[c * 64 + 2 * i + 1]);
                    tmem_st32(tS + c * 32, pk);
                }
            }
            const float2 lsum = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
            l += lsum.x + lsum.y;
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[wg]);
        }
        // Epilogue: O · v_scale[c] / l (FP8) or O / l (bf16) -> bf16 -> global.
        if (ok) ok = mbar_wait(&bars.o_ready[wg], (nkv - 1) & 1, abort_flag, err);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const int qrow = q0 + wg * kBM + row;
            __nv_bfloat16* orow = o + b * sb + h * sh + static_cast<int64_t>(qrow) * sn;
            const float* vsc = v_scale + static_cast<int64_t>(bh) * D;
            uint32_t ro[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tO + c * 32, ro);
                tmem_wait_ld();
                reg_fence32(ro);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float f0 = __uint_as_float(ro[2 * i]) * inv_l, f1 = __uint_as_float(ro[2 * i + 1]) * inv_l;
                    if (FP8) {
                        f0 *= __ldg(vsc + c * 32 + 2 * i);
                        f1 *= __ldg(vsc + c * 32 + 2 * i + 1);
                    }
                    pk[i] = pack_bf16x2(f0, f1);
                }
                if (qrow < N) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <bool FP8, int D>
cudaError_t launch_mode(const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv, const uint8_t* ws,
                        const Q8Layout& L, void* o, int64_t sb, int64_t sh, int64_t sn, int B, int H, int N,
                        float scale_log2, int* err, cudaStream_t stream) {
    using C = Q8Cfg<FP8, D>;
    static_assert(C::kSmemBytes <= 232448, "shared memory budget");
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_q8_kernel<FP8, D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_fwd_q8_kernel<FP8, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int n_pairs = ((N + kBM - 1) / kBM + 1) / 2;
    const int64_t grid = static_cast<int64_t>(B) * H * n_pairs;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    attn_fwd_q8_kernel<FP8, D><<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(
        tq8, tk8, tv, reinterpret_cast<const float*>(ws + L.q_scale), reinterpret_cast<const float*>(ws + L.k_scale),
        reinterpret_cast<const float*>(ws + L.v_scale), static_cast<__nv_bfloat16*>(o), sb, sh, sn, H, N, n_pairs,
        scale_log2, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_q8(const CUtensorMap& tq8, const CUtensorMap& tk8, const CUtensorMap& tv, int pv_fp8,
                           const uint8_t* ws, const Q8Layout& L, void* o, int64_t sb, int64_t sh, int64_t sn, int B,
                           int H, int N, int d, float scale_log2, int* err, cudaStream_t stream) {
    if (d == 128) {
        if (pv_fp8) return launch_mode<true, 128>(tq8, tk8, tv, ws, L, o, sb, sh, sn, B, H, N, scale_log2, err, stream);
        return launch_mode<false, 128>(tq8, tk8, tv, ws, L, o, sb, sh, sn, B, H, N, scale_log2, err, stream);
    }
    if (d == 64) {
        if (pv_fp8) return launch_mode<true, 64>(tq8, tk8, tv, ws, L, o, sb, sh, sn, B, H, N, scale_log2, err, stream);
        return launch_mode<false, 64>(tq8, tk8, tv, ws, L, o, sb, sh, sn, B, H, N, scale_log2, err, stream);
    }
    return cudaErrorInvalidValue;
}

}  // namespace ditk
