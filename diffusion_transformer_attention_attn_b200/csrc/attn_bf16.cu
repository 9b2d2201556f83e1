// Softmax attention O = softmax(scale · Q Kᵀ) V for bf16 [B, H, N, d] tensors
// on sm_100a: TMA-staged tiles, tcgen05 MMAs accumulating in tensor memory,
// and an exp2 online softmax with a running row max and row sum.
//
// What is computed follows "Flash Attention 2 accelerates Z-Image S3-DiT 6B"
// (opening section): one joint token stream, no mask, QKᵀ, softmax and V
// evaluated tile by tile in on-chip memory so the N×N logits never reach HBM.
//
// Work unit: one CTA takes 256 query rows (two 128-row tiles, "Q0" and "Q1")
// of one (b, h) and sweeps all keys in 128-key tiles.  Warp roles:
//   warps 0-3  softmax for Q0 (one thread per query row)
//   warps 4-7  softmax for Q1
//   warp  8    TMA producer (Q once, then a ring of K and V tiles)
//   warp  9    MMA issuer (one elected lane)
//   warps 10-11 complete the third warpgroup (idle)
// Registers: launched at 168 per thread; the producer warpgroup drops to 72
// and the two softmax warpgroups rise to 216 (2·128·216 + 128·72 = 384·168).
// (At 224/56 the producer and MMA warps spilled; 216/72 is spill-free and 3%
// faster.)
// Tensor memory (512 columns × 128 lanes × 32 bit):
//   [0,128)  S0 = Q0·Kᵀ (fp32); after the softmax, P0 (bf16 pairs) in [0,64),
//            written and published in two 64-key halves (kSplitP)
//   [128,256) S1 / P1
//   [256,256+d) O0 accumulator;  [256+d, 256+2d) O1 accumulator
// The MMA warp alternates the two tiles so that the tensor core computes
// P1·V and the next Q1·Kᵀ while the Q0 softmax runs, and vice versa.
//
// Online softmax (per row, in log2 units t = s·scale·log2 e): the running max
// m only moves when a new tile's max exceeds it by more than 8 (a factor 256
// in P); only then is the O row in tensor memory rescaled by 2^(m_old-m_new)
// and the row sum l with it.  P = 2^(t - m) ≤ 256 is exact enough in bf16
// and O, l are fp32.  Keys at or past N (the ragged last tile, zero-filled
// by TMA) get t = -inf, hence P = 0.
//
// Queries and keys may have different lengths (Nq rows against Nkv keys), so
// one launch can cover one chunk of a longer key sequence.  With `lse` given,
// each row also stores its log-sum-exp, ln Σ_j exp(scale·s_j) =
// ln 2 · (m + log2 l), the quantity that lets the outputs of several key
// chunks be merged into the attention over all of them (dit_attn_merge).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "internal.h"
#include "sm100_ptx.cuh"

// The softmax reads its logits through a lambda that captures the register
// array before tcgen05.ld fills it; every read comes after the load and its
// wait, so the front end's "used before its value is set" note is spurious.
#pragma nv_diag_suppress 549

namespace ditk {
namespace {

constexpr int kBM = 128;          // query rows per tile
constexpr int kBN = 128;          // keys per tile
constexpr int kThreads = 384;     // 12 warps (3 warpgroups)
constexpr int kLaunchRegs = 168;  // registers per thread the launch must provide
constexpr int kSoftmaxRegs = 216;
constexpr int kOtherRegs = 72;
// Pairs of exponentials (out of every 8) evaluated on the FMA pipe.
constexpr int kEmuOf8 = 1;
// Publish P in two 64-key halves (the MMA warp starts P·V on the first half
// while the second is computed) or whole.  Halves measured 2% faster.
constexpr bool kSplitP = true;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
constexpr int kLoadWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kHalfBytes = 128 * 128;  // one TMA box: 128 rows × 64 bf16 (128 B, swizzled)

template <int D>
struct Cfg {
    static constexpr int kTileBytes = kBM * D * 2;            // 128 rows × d bf16
    static constexpr int kHalves = D / 64;                    // 64-element swizzle atoms along d
    static constexpr int kStages = (D == 128) ? 2 : 4;        // K ring depth == V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kKOff = 2 * kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    // barriers: q_full, k_full[S], k_empty[S], v_full[S], v_empty[S],
    //           s_full[2], p_full[2 tiles × 2 halves], o_ready[2], mma_done
    static constexpr int kNumBars = 1 + 4 * kStages + 8 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;    // + slack for 1024-B alignment
    // S tiles: M=128 rows, N=128 keys, K-major A (Q) and B (K).
    static constexpr uint32_t kIdescQK = make_idesc(1, 1, 1, 0, 0, 128, kBN);
    // O += P·V: A = P from TMEM (K-major), B = V with d contiguous (MN-major).
    static constexpr uint32_t kIdescPV = make_idesc(1, 1, 1, 0, 1, 128, D);
};

struct Bars {
    uint64_t* q_full;
    uint64_t* k_full;
    uint64_t* k_empty;
    uint64_t* v_full;
    uint64_t* v_empty;
    uint64_t* s_full;
    uint64_t* p_full;
    uint64_t* o_ready;
    uint64_t* mma_done;
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
    using C = Cfg<D>;
    uint64_t* b = reinterpret_cast<uint64_t*>(base + C::kBarOff);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + C::kStages;
    r.v_full = r.k_empty + C::kStages;
    r.v_empty = r.v_full + C::kStages;
    r.s_full = r.v_empty + C::kStages;
    r.p_full = r.s_full + 2;
    r.o_ready = r.p_full + 4;
    r.mma_done = r.o_ready + 2;
    return r;
}

// K-major operand (Q or K tile, 128-B swizzle, SBO = 8 rows × 128 B) at
// k-step kk (16 bf16 along d): the d-halves are separate 16 KB panels;
// inside a panel, +32 B per k-step.
__host__ __device__ constexpr uint32_t kmajor_off(int kk) { return (kk >> 2) * kHalfBytes + (kk & 3) * 32; }
// MN-major V tile (LBO = distance between the 64-wide d panels, SBO = 8 keys ×
// 128 B) at key-step kk (16 keys): +16 rows × 128 B.
__host__ __device__ constexpr uint32_t v_off(int kk) { return kk * 16 * 128; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_bf16_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv, __nv_bfloat16* __restrict__ o, int64_t sb,
                         int64_t sh, int64_t sn, int H, int Nq, int Nkv, int n_pairs, float scale_log2,
                         float* __restrict__ lse, int* err) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Bars bars = carve_bars<D>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    const int pair = blockIdx.x % n_pairs;
    const int bh = blockIdx.x / n_pairs;
    const int b = bh / H;
    const int h = bh % H;
    const int q0 = pair * 2 * kBM;
    const int nkv = (Nkv + kBN - 1) / kBN;

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
            mbar_init(&bars.p_full[2 * t], kBM);
            mbar_init(&bars.p_full[2 * t + 1], kBM);
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
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tq);
            tma_prefetch_desc(&tk);
            tma_prefetch_desc(&tv);
            mbar_arrive_expect_tx(bars.q_full, 2 * C::kTileBytes);
            for (int t = 0; t < 2; ++t)
                for (int hf = 0; hf < C::kHalves; ++hf)
                    tma_load_4d(smem + C::kQOff + t * C::kTileBytes + hf * kHalfBytes, &tq, bars.q_full, hf * 64,
                                q0 + t * kBM, h, b);
        }
        __syncwarp();
        int nk[C::kStages], nv[C::kStages];  // times each stage was armed
#pragma unroll
        for (int s = 0; s < C::kStages; ++s) nk[s] = nv[s] = 0;
        for (int j = 0; j < nkv; ++j) {
            const int s = j % C::kStages;
            const uint32_t ph = (j / C::kStages) & 1;
            if (j >= C::kStages && !mbar_wait_lean(&bars.k_empty[s], ph ^ 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars.k_full[s], C::kTileBytes);
                for (int hf = 0; hf < C::kHalves; ++hf)
                    tma_load_4d(smem + C::kKOff + s * C::kTileBytes + hf * kHalfBytes, &tk, &bars.k_full[s],
                                hf * 64, j * kBN, h, b);
            }
            __syncwarp();
            ++nk[s];
            if (j >= C::kStages && !mbar_wait_lean(&bars.v_empty[s], ph ^ 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&bars.v_full[s], C::kTileBytes);
                for (int hf = 0; hf < C::kHalves; ++hf)
                    tma_load_4d(smem + C::kVOff + s * C::kTileBytes + hf * kHalfBytes, &tv, &bars.v_full[s],
                                hf * 64, j * kBN, h, b);
            }
            __syncwarp();
            ++nv[s];
        }
        if (*abort_flag && lane == 0) {
            // Let every copy this warp started land before the CTA can exit:
            // the n-th arming of a stage completes that barrier's phase n-1.
            mbar_wait_drain(bars.q_full, 0);
            for (int s = 0; s < C::kStages; ++s) {
                if (nk[s] > 0) mbar_wait_drain(&bars.k_full[s], (nk[s] - 1) & 1);
                if (nv[s] > 0) mbar_wait_drain(&bars.v_full[s], (nv[s] - 1) & 1);
            }
        }
      } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        const SDesc dQ0 = sdesc_sw128(smem_base + C::kQOff, 16, 1024);
        const SDesc dQ1 = sdesc_add(dQ0, C::kTileBytes);
        const SDesc dK0 = sdesc_sw128(smem_base + C::kKOff, 16, 1024);
        const SDesc dV0 = sdesc_sw128(smem_base + C::kVOff, kHalfBytes, 1024);
        const uint32_t tS0 = tmem, tS1 = tmem + 128;
        const uint32_t tO0 = tmem + 256, tO1 = tmem + 256 + D;
        auto issue_s = [&](uint32_t tS, SDesc dQ, SDesc dK) {
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
                mma_ss<0>(tS, sdesc_add(dQ, kmajor_off(kk)), sdesc_add(dK, kmajor_off(kk)), C::kIdescQK, kk > 0);
        };
        bool ok = mbar_wait_lean(bars.q_full, 0, abort_flag, err) &&
                  mbar_wait_lean(&bars.k_full[0], 0, abort_flag, err);
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
                const SDesc dV = sdesc_add(dV0, vs * C::kTileBytes);
                const bool more = j + 1 < nkv;
                const int ks = (j + 1) % C::kStages;
                const SDesc dK = sdesc_add(dK0, ks * C::kTileBytes);
                ok = mbar_wait_lean(&bars.v_full[vs], (j / C::kStages) & 1, abort_flag, err);
                if (!ok) break;
                // O_t += P_t·V (in two 64-key halves when P is published in halves).
                auto issue_pv = [&](int t, uint32_t tO, uint32_t tP) {
                    constexpr int kParts = kSplitP ? 2 : 1;
#pragma unroll
                    for (int hf = 0; hf < kParts; ++hf) {
                        ok = ok && mbar_wait_lean(&bars.p_full[2 * t + hf], j & 1, abort_flag, err);
                        if (!ok) return;
                        tc_fence_after();
#pragma unroll
                        for (int kk = hf * (8 / kParts); kk < (hf + 1) * (8 / kParts); ++kk)
                            mma_ts<0>(tO, tP + kk * 8, sdesc_add(dV, v_off(kk)), C::kIdescPV, (j > 0 || kk > 0));
                        __syncwarp();
                    }
                };
                issue_pv(0, tO0, tS0);
                if (!ok) break;
                mma_commit(&bars.o_ready[0]);
                __syncwarp();
                if (more) {
                    ok = mbar_wait_lean(&bars.k_full[ks], ((j + 1) / C::kStages) & 1, abort_flag, err);
                    if (!ok) break;
                    tc_fence_after();
                    issue_s(tS0, dQ0, dK);
                    mma_commit(&bars.s_full[0]);
                    __syncwarp();
                }
                issue_pv(1, tO1, tS1);
                if (!ok) break;
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
        // Every MMA issued above has completed once mma_done flips.
        mma_commit(bars.mma_done);
        if (lane == 0) mbar_wait_drain(bars.mma_done, 0);
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        regs_inc<kSoftmaxRegs>();
        const int wg = warp >> 2;  // which query tile
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_off + wg * 128;
        const uint32_t tO = tmem + lane_off + 256 + wg * D;
        float m = -INFINITY;
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            ok = mbar_wait_lean(&bars.s_full[wg], j & 1, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            uint32_t r[kBN / 32][32];
            auto X = [&](int col) { return __uint_as_float(r[col >> 5][col & 31]); };
            const int valid = Nkv - j * kBN;  // keys of this tile below Nkv
            // Row max over the tile; keys past N are left out.  Full tiles load
            // S in 32-column chunks and fold each chunk into 8 independent
            // 3-input max chains while the next chunk is in flight.
            float tmax;
            if (valid >= kBN) {
                float mx[8];
                tmem_ld32(tS, r[0]);
                tmem_wait_ld();
                reg_fence32(r[0]);
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) {
                    if (c + 1 < kBN / 32) tmem_ld32(tS + (c + 1) * 32, r[c + 1]);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float a = X(c * 32 + i), b2 = X(c * 32 + 8 + i), c3 = X(c * 32 + 16 + i),
                                    d4 = X(c * 32 + 24 + i);
                        mx[i] = c == 0 ? fmax3(a, b2, fmaxf(c3, d4)) : fmax3(mx[i], fmax3(a, b2, c3), d4);
                    }
                    if (c + 1 < kBN / 32) {
                        tmem_wait_ld();
                        reg_fence32(r[c + 1]);
                    }
                }
                tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            } else {
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) tmem_ld32(tS + c * 32, r[c]);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < kBN / 32; ++c) reg_fence32(r[c]);
                tmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < kBN; ++c)
                    if (c < valid) tmax = fmaxf(tmax, X(c));
            }
            const float m_new = fmaxf(m, tmax * scale_log2);
            if (j == 0) {
                m = m_new;
            } else {
                const bool need = m_new > m + 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    // O holds P_{<j}·V; rescale it once P_{j-1}·V has landed.
                    ok = mbar_wait_lean(&bars.o_ready[wg], (j - 1) & 1, abort_flag, err);
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
            // P = 2^(s·scale·log2e − m): packed FFMA, ex2 (MUFU, or the FMA
            // pipe for kEmuOf8 pairs in 8), packed row sum, bf16 pairs into
            // tensor memory, one 64-key half at a time.  With kSplitP each half
            // is published as soon as it is written (its P·V MMAs then start
            // while the next half is computed); otherwise P is published once
            // whole.  Keys past N get P = 0.
            const float2 c2 = make_float2(scale_log2, scale_log2);
            const float2 negm2 = make_float2(-m, -m);
            float2 ls[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
            auto exp_half = [&](int hf, auto tail_tag) {
                constexpr bool kTail = decltype(tail_tag)::value;
                uint32_t p[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = hf * 64 + 2 * i;
                    const float2 t = __ffma2_rn(make_float2(X(col), X(col + 1)), c2, negm2);
                    float2 e;
                    if (!kTail && (i & 7) < kEmuOf8)
                        e = exp2_poly2(t);
                    else
                        e = make_float2(ex2_approx(t.x), ex2_approx(t.y));
                    if (kTail) {
                        if (col >= valid) e.x = 0.f;
                        if (col + 1 >= valid) e.y = 0.f;
                    }
                    ls[i & 3] = __fadd2_rn(ls[i & 3], e);
                    p[i] = pack_bf16x2(e.x, e.y);
                }
                tmem_st32(tS + hf * 32, p);
                if (kSplitP || hf == 1) {
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bars.p_full[2 * wg + (kSplitP ? hf : 0)]);
                }
            };
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                if (valid < kBN)
                    exp_half(hf, std::true_type{});
                else
                    exp_half(hf, std::false_type{});
            }
            const float2 lsum = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
            l += lsum.x + lsum.y;
        }
        // Epilogue: O / l -> bf16 -> global (rows at or past Nq are padding).
        if (ok) ok = mbar_wait_lean(&bars.o_ready[wg], (nkv - 1) & 1, abort_flag, err);
        if (ok) {
            tc_fence_after();
            const float inv_l = 1.0f / l;
            const int qrow = q0 + wg * kBM + row;
            __nv_bfloat16* orow = o + b * sb + h * sh + static_cast<int64_t>(qrow) * sn;
            uint32_t r[32];
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                tmem_ld32(tO + c * 32, r);
                tmem_wait_ld();
                reg_fence32(r);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    pk[i] = pack_bf16x2(__uint_as_float(r[2 * i]) * inv_l, __uint_as_float(r[2 * i + 1]) * inv_l);
                if (qrow < Nq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (lse != nullptr && qrow < Nq)
                lse[static_cast<int64_t>(bh) * Nq + qrow] = (m + __log2f(l)) * 0.69314718055994531f;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, int64_t sb,
                     int64_t sh, int64_t sn, int B, int H, int Nq, int Nkv, float scale_log2, float* lse, int* err,
                     cudaStream_t stream) {
    using C = Cfg<D>;
    static_assert(C::kSmemBytes <= 232448, "shared memory budget");
    // The register split inside the kernel needs the full launch allotment.
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_bf16_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_fwd_bf16_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int n_qt = (Nq + kBM - 1) / kBM;
    const int n_pairs = (n_qt + 1) / 2;
    const int64_t grid = static_cast<int64_t>(B) * H * n_pairs;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    attn_fwd_bf16_kernel<D><<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(
        tq, tk, tv, static_cast<__nv_bfloat16*>(o), sb, sh, sn, H, Nq, Nkv, n_pairs, scale_log2, lse, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                             int64_t sb, int64_t sh, int64_t sn, int B, int H, int Nq, int Nkv, int d,
                             float scale_log2, float* lse, int* err, cudaStream_t stream) {
    if (d == 128) return launch_d<128>(tq, tk, tv, o, sb, sh, sn, B, H, Nq, Nkv, scale_log2, lse, err, stream);
    if (d == 64) return launch_d<64>(tq, tk, tv, o, sb, sh, sn, B, H, Nq, Nkv, scale_log2, lse, err, stream);
    return cudaErrorInvalidValue;
}

}  // namespace ditk
