// Softmax attention O = softmax(scale · Q Kᵀ) V for bf16 tensors on sm_100a,
// one 128-row query tile per CTA with the keys of every tile split between two
// softmax warpgroups ("key-split" schedule).
//
// What is computed follows "Flash Attention 2 accelerates Z-Image S3-DiT 6B"
// (opening section): one joint token stream, no mask, QKᵀ, softmax and V
// evaluated tile by tile in on-chip memory.  The log-sum-exp output serves the
// key-chunk merge of "ParaAttention" (diffusers docs), "Context Parallelism".
//
// Schedule.  Each CTA owns 128 query rows of one (b, h) and sweeps the keys in
// 128-key tiles.  S(j) = Q·K(j)ᵀ lands in one of two tensor-memory buffers, so
// the tensor core computes S(j+1) while the softmax works on S(j).  Keys
// [0, 64) of every tile belong to warpgroup A, keys [64, 128) to warpgroup B;
// each keeps its own running max m, row sum l and output accumulator
// (O_A, O_B), like two independent attentions over interleaved key halves, so
// the two never exchange anything per tile.  The epilogue merges them once:
//   M = max(m_A, m_B),  O = (2^(m_A−M) O_A + 2^(m_B−M) O_B) / (2^(m_A−M) l_A + 2^(m_B−M) l_B).
// Warp roles (384 threads):
//   warps 0-3   softmax A (one thread per query row, keys [0,64) of each tile)
//   warps 4-7   softmax B (keys [64,128))
//   warp  8     TMA producer of Q and the K ring
//   warp  9     MMA issuer (one elected lane)
//   warp  10    TMA producer of the V ring
//   warp  11    idle
// Tensor memory (512 columns): S buffers [0,128) and [128,256) (fp32; after
// the softmax, P_A as bf16 pairs in the buffer's columns [0,32) and P_B in
// [64,96)), O_A [256, 256+d), O_B [256+d, 256+2d).
// Online softmax per warpgroup and row, in log2 units t = s·scale·log2 e: the
// running max moves only when a tile's max passes it by more than 8, and only
// then is that warpgroup's O row rescaled in tensor memory.  Keys at or past
// Nkv get P = 0.
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

constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = 128;          // keys per tile
constexpr int kHalfN = 64;        // keys per warpgroup per tile
constexpr int kThreads = 384;
constexpr int kLaunchRegs = 168;
constexpr int kSoftmaxRegs = 224;
constexpr int kOtherRegs = 56;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= kThreads * kLaunchRegs, "register split");
// Pairs of exponentials (out of every 8) evaluated on the FMA pipe.
constexpr int kEmuOf8 = 1;
constexpr int kKWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kVWarp = 10;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kHalfBytes = 128 * 128;  // one TMA box: 128 rows × 64 bf16 (128 B, swizzled)

template <int D>
struct Cfg {
    static constexpr int kTileBytes = kBM * D * 2;     // 128 rows × d bf16
    static constexpr int kHalves = D / 64;             // 64-element swizzle panels along d
    static constexpr int kKStages = (D == 128) ? 3 : 4;
    static constexpr int kVStages = (D == 128) ? 3 : 4;
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kTileBytes;
    static constexpr int kVOff = kKOff + kKStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kVStages * kTileBytes;
    // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS],
    //           s_full[2 buffers], p_full[2 warpgroups × 2 buffers], o_ready[2 warpgroups], mma_done
    static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 4 + 2 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kSmemBytes = kMiscOff + 64 + 1024;  // + slack for 1024-B alignment
    static constexpr uint32_t kIdescQK = make_idesc(1, 1, 1, 0, 0, 128, kBN);
    static constexpr uint32_t kIdescPV = make_idesc(1, 1, 1, 0, 1, 128, D);
};

struct Bars {
    uint64_t* q_full;
    uint64_t* k_full;
    uint64_t* k_empty;
    uint64_t* v_full;
    uint64_t* v_empty;
    uint64_t* s_full;   // [buffer]
    uint64_t* p_full;   // [2 * warpgroup + buffer]
    uint64_t* o_ready;  // [warpgroup]
    uint64_t* mma_done;
};

template <int D>
__device__ __forceinline__ Bars carve_bars(uint8_t* base) {
    using C = Cfg<D>;
    uint64_t* b = reinterpret_cast<uint64_t*>(base + C::kBarOff);
    Bars r;
    r.q_full = b;
    r.k_full = b + 1;
    r.k_empty = r.k_full + C::kKStages;
    r.v_full = r.k_empty + C::kKStages;
    r.v_empty = r.v_full + C::kVStages;
    r.s_full = r.v_empty + C::kVStages;
    r.p_full = r.s_full + 2;
    r.o_ready = r.p_full + 4;
    r.mma_done = r.o_ready + 2;
    return r;
}

// K-major operand (Q or K tile) at k-step kk (16 bf16 along d): the d-halves
// are separate 16 KB panels; inside a panel, +32 B per k-step.
__host__ __device__ constexpr uint32_t kmajor_off(int kk) { return (kk >> 2) * kHalfBytes + (kk & 3) * 32; }
// MN-major V tile at key-step kk (16 keys): +16 rows × 128 B.
__host__ __device__ constexpr uint32_t v_off(int kk) { return kk * 16 * 128; }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_bf16_ks_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                            const __grid_constant__ CUtensorMap tv, __nv_bfloat16* __restrict__ o, int64_t sb,
                            int64_t sh, int64_t sn, int H, int Nq, int Nkv, int n_qt, float scale_log2,
                            float* __restrict__ lse, int* err) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const Bars bars = carve_bars<D>(smem);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qt = blockIdx.x % n_qt;
    const int bh = blockIdx.x / n_qt;
    const int b = bh / H;
    const int h = bh % H;
    const int q0 = qt * kBM;
    const int nkv = (Nkv + kBN - 1) / kBN;

    if (threadIdx.x == 0) {
        mbar_init(bars.q_full, 1);
        for (int s = 0; s < C::kKStages; ++s) {
            mbar_init(&bars.k_full[s], 1);
            mbar_init(&bars.k_empty[s], 1);
        }
        for (int s = 0; s < C::kVStages; ++s) {
            mbar_init(&bars.v_full[s], 1);
            mbar_init(&bars.v_empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&bars.s_full[i], 1);
            mbar_init(&bars.o_ready[i], 1);
        }
        for (int i = 0; i < 4; ++i) mbar_init(&bars.p_full[i], kBM);
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
      if (warp == kKWarp || warp == kVWarp) {
        // ------------------------------------------------------------ TMA producers
        const bool is_k = (warp == kKWarp);
        const CUtensorMap* map = is_k ? &tk : &tv;
        uint64_t* full = is_k ? bars.k_full : bars.v_full;
        uint64_t* empty = is_k ? bars.k_empty : bars.v_empty;
        const int stages = is_k ? C::kKStages : C::kVStages;
        const int off = is_k ? C::kKOff : C::kVOff;
        if (lane == 0) {
            tma_prefetch_desc(map);
            if (is_k) {
                tma_prefetch_desc(&tq);
                mbar_arrive_expect_tx(bars.q_full, C::kTileBytes);
                for (int hf = 0; hf < C::kHalves; ++hf)
                    tma_load_4d(smem + C::kQOff + hf * kHalfBytes, &tq, bars.q_full, hf * 64, q0, h, b);
            }
        }
        __syncwarp();
        int armed[4] = {0, 0, 0, 0};  // times each stage was armed
        for (int j = 0; j < nkv; ++j) {
            const int s = j % stages;
            const uint32_t ph = (j / stages) & 1;
            if (j >= stages && !mbar_wait(&empty[s], ph ^ 1, abort_flag, err)) break;
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], C::kTileBytes);
                for (int hf = 0; hf < C::kHalves; ++hf)
                    tma_load_4d(smem + off + s * C::kTileBytes + hf * kHalfBytes, map, &full[s], hf * 64, j * kBN, h,
                                b);
            }
            __syncwarp();
            ++armed[s];
        }
        if (*abort_flag && lane == 0) {
            // Let every copy this warp started land before the CTA can exit:
            // the n-th arming of a stage completes that barrier's phase n-1.
            if (is_k) mbar_wait_drain(bars.q_full, 0);
            for (int s = 0; s < stages; ++s)
                if (armed[s] > 0) mbar_wait_drain(&full[s], (armed[s] - 1) & 1);
        }
      } else if (warp == kMmaWarp) {
        // ------------------------------------------------------------ MMA issuer
        const SDesc dQ = sdesc_sw128(smem_base + C::kQOff, 16, 1024);
        const SDesc dK0 = sdesc_sw128(smem_base + C::kKOff, 16, 1024);
        const SDesc dV0 = sdesc_sw128(smem_base + C::kVOff, kHalfBytes, 1024);
        const uint32_t tOA = tmem + 256, tOB = tmem + 256 + D;
        bool ok = mbar_wait(bars.q_full, 0, abort_flag, err);
        // S(j) = Q·K(j)ᵀ into buffer j % 2; releases K stage j % KS.
        auto issue_s = [&](int j) -> bool {
            const int ks = j % C::kKStages;
            if (!mbar_wait(&bars.k_full[ks], (j / C::kKStages) & 1, abort_flag, err)) return false;
            tc_fence_after();
            {
                const SDesc dK = sdesc_add(dK0, ks * C::kTileBytes);
                const uint32_t tS = tmem + (j & 1) * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    mma_ss<0>(tS, sdesc_add(dQ, kmajor_off(kk)), sdesc_add(dK, kmajor_off(kk)), C::kIdescQK, kk > 0);
                mma_commit(&bars.s_full[j & 1]);
                mma_commit(&bars.k_empty[ks]);
            }
            __syncwarp();
            return true;
        };
        if (ok) ok = issue_s(0);
        if (ok && nkv > 1) ok = issue_s(1);
        for (int j = 0; j < nkv && ok; ++j) {
            const int vs = j % C::kVStages;
            const int buf = j & 1;
            ok = mbar_wait(&bars.v_full[vs], (j / C::kVStages) & 1, abort_flag, err);
            if (!ok) break;
            const SDesc dV = sdesc_add(dV0, vs * C::kTileBytes);
            // O_g += P_g(j)·V(j)[keys of g], once warpgroup g has published P_g(j).
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                ok = mbar_wait(&bars.p_full[2 * g + buf], (j >> 1) & 1, abort_flag, err);
                if (!ok) break;
                tc_fence_after();
                {
                    const uint32_t tP = tmem + buf * 128 + g * kHalfN;
                    const uint32_t tO = g == 0 ? tOA : tOB;
#pragma unroll
                    for (int kk = 0; kk < kHalfN / 16; ++kk)
                        mma_ts<0>(tO, tP + kk * 8, sdesc_add(dV, v_off(g * (kHalfN / 16) + kk)), C::kIdescPV,
                                  (j > 0 || kk > 0));
                    mma_commit(&bars.o_ready[g]);
                }
                __syncwarp();
            }
            if (!ok) break;
            mma_commit(&bars.v_empty[vs]);
            __syncwarp();
            // S(j+2) reuses buffer j % 2, whose P(j) the MMAs above read first.
            if (j + 2 < nkv) ok = issue_s(j + 2);
        }
        // Every MMA issued above has completed once mma_done flips.
        mma_commit(bars.mma_done);
        if (lane == 0) mbar_wait_drain(bars.mma_done, 0);
        __syncwarp();
      }
    } else {
        // ------------------------------------------------------------ softmax (warps 0-7)
        regs_inc<kSoftmaxRegs>();
        const int g = warp >> 2;  // 0: keys [0,64) of each tile, 1: keys [64,128)
        const int row = (warp & 3) * 32 + lane;
        const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
        const uint32_t tO = tmem + lane_off + 256 + g * D;
        float m = -INFINITY;
        float l = 0.f;
        bool ok = true;
        for (int j = 0; j < nkv; ++j) {
            const int buf = j & 1;
            ok = mbar_wait(&bars.s_full[buf], (j >> 1) & 1, abort_flag, err);
            if (!ok) break;
            tc_fence_after();
            const uint32_t tS = tmem + lane_off + buf * 128 + g * kHalfN;
            uint32_t r[kHalfN / 32][32];
            auto X = [&](int col) { return __uint_as_float(r[col >> 5][col & 31]); };
            const int valid = Nkv - j * kBN - g * kHalfN;  // keys of this half below Nkv (may be <= 0)
            tmem_ld32(tS, r[0]);
            tmem_ld32(tS + 32, r[1]);
            tmem_wait_ld();
            reg_fence32(r[0]);
            reg_fence32(r[1]);
            float tmax;
            if (valid >= kHalfN) {
                float mx[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    mx[i] = fmax3(fmax3(X(i), X(8 + i), X(16 + i)), fmax3(X(24 + i), X(32 + i), X(40 + i)),
                                  fmaxf(X(48 + i), X(56 + i)));
                tmax = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            } else {
                tmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < kHalfN; ++c)
                    if (c < valid) tmax = fmaxf(tmax, X(c));
            }
            const float m_new = fmaxf(m, tmax * scale_log2);
            if (j == 0) {
                m = m_new;
            } else {
                const bool need = m_new > m + 8.0f;
                if (__any_sync(0xffffffffu, need)) {
                    // O_g holds P_g(<j)·V; rescale it once P_g(j-1)·V has landed.
                    ok = mbar_wait(&bars.o_ready[g], (j - 1) & 1, abort_flag, err);
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
            // P = 2^(s·scale·log2e − m) for this half's 64 keys: packed FFMA,
            // ex2 (MUFU, or the FMA pipe for kEmuOf8 pairs in 8), packed row
            // sum, bf16 pairs into the first 32 columns of this half.  A row
            // that has seen no key yet (m = -inf) gets P = 0.
            const float2 c2 = make_float2(scale_log2, scale_log2);
            const float mm = (m == -INFINITY) ? 0.f : m;
            const float2 negm2 = make_float2(-mm, -mm);
            float2 ls[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) ls[i] = make_float2(0.f, 0.f);
            auto exps = [&](auto tail_tag) {
                constexpr bool kTail = decltype(tail_tag)::value;
                uint32_t p[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int col = 2 * i;
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
                tmem_st32(tS, p);
            };
            if (valid >= kHalfN && m != -INFINITY)
                exps(std::false_type{});
            else
                exps(std::true_type{});
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars.p_full[2 * g + buf]);
            const float2 lsum = __fadd2_rn(__fadd2_rn(ls[0], ls[1]), __fadd2_rn(ls[2], ls[3]));
            l += lsum.x + lsum.y;
        }
        // Epilogue.  Both accumulators are final once the last P·V of each
        // warpgroup has landed.  The two threads of a row swap (m, l) through
        // shared memory (the Q tile's space, no longer read by any MMA), then
        // each writes half of the row's d columns.
        bool fin = ok;
        if (fin) fin = mbar_wait(&bars.o_ready[0], (nkv - 1) & 1, abort_flag, err);
        if (fin) fin = mbar_wait(&bars.o_ready[1], (nkv - 1) & 1, abort_flag, err);
        float* xch = reinterpret_cast<float*>(smem + C::kQOff);  // [2 warpgroups][2 values][128 rows]
        if (fin) {
            xch[(g * 2 + 0) * kBM + row] = m;
            xch[(g * 2 + 1) * kBM + row] = l;
        }
        // Named barrier 1 over the 256 softmax threads (every one of them
        // reaches it: the waits above are bounded and never return early).
        asm volatile("bar.sync 1, 256;" ::: "memory");
        fin = fin && (*abort_flag == 0);
        if (fin) {
            tc_fence_after();
            const float mA = xch[0 * kBM + row], lA = xch[1 * kBM + row];
            const float mB = xch[2 * kBM + row], lB = xch[3 * kBM + row];
            const float M = fmaxf(mA, mB);
            const float wA = ex2_approx(mA - M), wB = (mB == -INFINITY) ? 0.f : ex2_approx(mB - M);
            const float L = wA * lA + wB * lB;
            const float fA = wA / L, fB = wB / L;
            const int qrow = q0 + row;
            __nv_bfloat16* orow = o + b * sb + h * sh + static_cast<int64_t>(qrow) * sn + g * (D / 2);
            const uint32_t tA = tmem + lane_off + 256 + g * (D / 2);
            const uint32_t tB = tA + D;
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t ra[32], rb[32];
                tmem_ld32(tA + c * 32, ra);
                tmem_ld32(tB + c * 32, rb);
                tmem_wait_ld();
                reg_fence32(ra);
                reg_fence32(rb);
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float x0 = __uint_as_float(ra[2 * i]) * fA + __uint_as_float(rb[2 * i]) * fB;
                    const float x1 = __uint_as_float(ra[2 * i + 1]) * fA + __uint_as_float(rb[2 * i + 1]) * fB;
                    pk[i] = pack_bf16x2(x0, x1);
                }
                if (qrow < Nq) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            if (lse != nullptr && g == 0 && qrow < Nq)
                lse[static_cast<int64_t>(bh) * Nq + qrow] = (M + __log2f(L)) * 0.69314718055994531f;
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
cudaError_t launch_ks_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, int64_t sb,
                        int64_t sh, int64_t sn, int B, int H, int Nq, int Nkv, float scale_log2, float* lse, int* err,
                        cudaStream_t stream) {
    using C = Cfg<D>;
    static_assert(C::kSmemBytes <= 232448, "shared memory budget");
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attn_fwd_bf16_ks_kernel<D>);
    if (e != cudaSuccess) return e;
    if (fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(attn_fwd_bf16_ks_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    const int n_qt = (Nq + kBM - 1) / kBM;
    const int64_t grid = static_cast<int64_t>(B) * H * n_qt;
    if (grid > 0x7FFFFFFF) return cudaErrorInvalidValue;
    attn_fwd_bf16_ks_kernel<D><<<static_cast<unsigned>(grid), kThreads, C::kSmemBytes, stream>>>(
        tq, tk, tv, static_cast<__nv_bfloat16*>(o), sb, sh, sn, H, Nq, Nkv, n_qt, scale_log2, lse, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_bf16_ks(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                                int64_t sb, int64_t sh, int64_t sn, int B, int H, int Nq, int Nkv, int d,
                                float scale_log2, float* lse, int* err, cudaStream_t stream) {
    if (d == 128) return launch_ks_d<128>(tq, tk, tv, o, sb, sh, sn, B, H, Nq, Nkv, scale_log2, lse, err, stream);
    if (d == 64) return launch_ks_d<64>(tq, tk, tv, o, sb, sh, sn, B, H, Nq, Nkv, scale_log2, lse, err, stream);
    return cudaErrorInvalidValue;
}

}  // namespace ditk
