// Tensor-core (tcgen05 + TMEM + TMA) prefill for the gated delta rule with
// bf16 inputs ("Efficient attention variants" §7.4):
//     S_t = alpha_t S_{t-1} + g_t k_t (v_t - alpha_t S_{t-1}^T k_t)^T,  o_t = S_t^T q_t
//
// Chunk form (a WY / UT representation, derived here; the pages give only the
// recurrence and the remark that chunked kernels pass state between chunks,
// "Efficient attention variants" §8).  For a chunk of C tokens with start
// state S, L_i = sum_{m<=i} log alpha_m, b_i = e^{L_i}:
//   every S_t in the chunk has the form  b_t S + sum_{j<=t} e^{L_t-L_j} k_j u_j^T
//   with pseudo-values u solving  (I + A) U = diag(g) (V - diag(b) K S),
//   A_tj = g_t e^{L_t-L_j} (k_t . k_j) for j < t (strictly lower).
// With T = (I + A)^{-1}, T' = T diag(g):
//   W = T' diag(b) K,  U = T' V - W S
//   O = diag(b) Q S + P~ U,   P~_tj = e^{L_t-L_j} (q_t . k_j) [j <= t]
//   S_next = b_C S + K~^T U,   K~ = diag(b_C / b) K
// Substituting back reproduces the token recurrence exactly (up to rounding).
//
// Only U and S_next depend on the state, so the work splits in two launches:
//   gd_prep_kernel   every (chain, chunk) in parallel: the score blocks
//                    [K;Q]K^T, A and P~, T = (I + A)^{-1} on the CUDA cores in
//                    fp32 (blocked forward substitution), T', W = T' diag(b) K.
//                    Writes -W, diag(b) Q, diag(b_C / b) K, T' and P~ (bf16) to
//                    the workspace.
//   gd_chain_kernel  one CTA per (chain, 64 value columns), chunks in order:
//                    U = T' V + (-W) S and diag(b) Q S, then P~ U and the state
//                    update, all on the tensor cores; the CUDA cores only
//                    convert U and S to bf16 operands, scale S by b_C and write
//                    the output.  A tcgen05.mma costs about the same to issue
//                    at M = 64 as at M = 128, so operands that share a B are
//                    stacked into M = 128: [T'; 0] V, [-W; diag(b) Q] S and
//                    [0; P~] U leave U in accumulator rows 0-63 and the whole
//                    output in rows 64-127.  Issue itself is slow (tens of
//                    cycles per MMA), so two warps issue, each half of every
//                    contraction on the chain into its own TMEM accumulator
//                    (the converters add the pair when they read it out); one
//                    also issues the next chunk's T' V, the other P~ U.
// The columns of S evolve independently under the delta rule, so value tiles
// need no communication.
#include <algorithm>
#include <cmath>

#include <cudaTypedefs.h>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int C = 64;            // tokens per chunk
constexpr int DVT = 64;          // value columns per chain-kernel CTA
constexpr int kThreads = 256;    // two warpgroups
constexpr int TILE = kTileBytes; // 64 rows x 128 bytes
// log alpha is clamped here so that alpha = 0 (a full reset) never forms inf - inf
constexpr float kLogAlphaMin = -80.f;

// fp32 -> tf32 (round to nearest, ties away) for the warp-level MMA below.
__device__ __forceinline__ uint32_t to_tf32(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D (16x8, fp32) += A (16x8, tf32, row-major) * B (8x8, tf32, column-major):
// the warp-level m16n8k8 MMA, used for the 16 x 16 block products of the
// triangular solve (too small to fill a tcgen05 tile).  Fragments: with
// g = lane / 4, t = lane % 4, a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]},
// b = {B[t][g], B[t+4][g]}, d = {D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]}.
__device__ __forceinline__ void mma_16x8x8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
                 "{%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Within-chunk inclusive log decay for the two tokens 2*lane, 2*lane + 1 of a
// chunk (one warp covers the chunk).  Tokens past the sequence end count as
// alpha = 1.  Returns L of both tokens and L_C of the chunk.
__device__ __forceinline__ void chunk_logdecay(float a0, float a1, bool ok0, bool ok1, int lane, float& La,
                                               float& Lb, float& Lc)
{
    const float l0 = ok0 ? fmaxf(__logf(a0), kLogAlphaMin) : 0.f;
    const float l1 = ok1 ? fmaxf(__logf(a1), kLogAlphaMin) : 0.f;
    float incl = l0 + l1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const float t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    La = incl - l1;
    Lb = incl;
    Lc = __shfl_sync(0xffffffffu, incl, 31);
}

// ===========================================================================
// gd_prep_kernel
// ===========================================================================

template <int D>
struct PrepPlan {
    static constexpr int NB = D / 64;                       // feature blocks
    // [K_0 Q_0 K_1 Q_1 ...]: K_b and Q_b adjacent form the M = 128 A operand of M1
    static constexpr int LOAD_BYTES = 2 * NB * TILE;
    static constexpr int OFF_KB = 2 * NB * TILE;            // diag(b) K, MN-major B of M2
    static constexpr int OFF_T = 3 * NB * TILE;             // T' bf16 [C][C]
    static constexpr int OFF_P = OFF_T + TILE;              // P~ bf16 [C][C]
    static constexpr int OFF_A = OFF_P + TILE;              // A fp32 [C][C+1]; later the -W staging tiles
    static constexpr int TS = C + 4;                        // row stride of T (16-byte aligned rows)
    static constexpr int OFF_TM = OFF_A + C * (C + 1) * 4;  // T fp32 [C][TS]
    static constexpr int OFF_X = OFF_TM + C * TS * 4;       // per-warp 16 x 8 block scratch, fp32 [8][16][9]
    // L[C], b[C], g[C], staged alpha/g [2][2][C], e^{L-L_m}[C], e^{L_m-L}[C], b_C/b[C], flag
    static constexpr int OFF_VEC = OFF_X + 8 * 16 * 9 * 4;
    static constexpr int OFF_BAR = OFF_VEC + 10 * C * 4 + 16;
    static constexpr int OFF_TMEM = OFF_BAR + 3 * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(NB * TILE <= C * (C + 1) * 4, "-W staging fits over A");
    static_assert(2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
    // TMEM columns: score blocks (rows 0-63 K K^T, 64-127 Q K^T), then W
    static constexpr uint32_t T_KQ = 0, T_W = 64, T_COLS = 256;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
gd_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_t,
               const __grid_constant__ CUtensorMap tm_p, const float* __restrict__ alpha,
               const float* __restrict__ gate, float* __restrict__ vec, int N, int chains, int ld)
{
    using P = PrepPlan<D>;
    constexpr int NB = P::NB;
    grid_launch_dependents();   // the chain kernel may launch; it waits for this grid's results
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* kbt = sm + P::OFF_KB;
    unsigned char* ttile = sm + P::OFF_T;
    unsigned char* ptile = sm + P::OFF_P;
    unsigned char* wstage = sm + P::OFF_A;
    float* As = reinterpret_cast<float*>(sm + P::OFF_A);
    float* Tm = reinterpret_cast<float*>(sm + P::OFF_TM);
    float* Xs = reinterpret_cast<float*>(sm + P::OFF_X);
    float* Lv = reinterpret_cast<float*>(sm + P::OFF_VEC);
    float* bv = Lv + C;
    float* gv = Lv + 2 * C;
    float* avec = Lv + 3 * C;   // [2][2][C]: alpha, g of two work items
    float* ef = Lv + 7 * C;     // e^{L_t - L_m}, m the chunk's middle token
    float* eg = Lv + 8 * C;     // e^{L_m - L_t}
    int* factored = reinterpret_cast<int*>(Lv + 10 * C);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* bar1 = full + 1;
    uint64_t* bar2 = full + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const int nch = (N + C - 1) / C;
    const int items = chains * nch;
    const uint64_t pol = policy_evict_first();

    if (tid == 0) {
        mbar_init(full, 1);
        mbar_init(bar1, 1);
        mbar_init(bar2, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    int loads_issued = 0, commits1 = 0, commits2 = 0;
    auto issue = [&](int item) {
        const int ch = item / nch, y = (item % nch) * C;
        mbar_expect_tx(full, P::LOAD_BYTES);
        for (int b = 0; b < NB; ++b) {
            tma_load_3d(sm + (2 * b) * TILE, &tm_k, b * 64, y, ch, full, pol);
            tma_load_3d(sm + (2 * b + 1) * TILE, &tm_q, b * 64, y, ch, full, pol);
        }
        ++loads_issued;
    };
    // warp 1: alpha, g of a work item into staging buffer `buf` (lane: tokens 2 lane, 2 lane + 1)
    auto stage_vectors = [&](int item, int buf) {
        const int ch = item / nch, t0 = (item % nch) * C;
        const float* al = alpha + (size_t)ch * ld;
        const float* gl = gate + (size_t)ch * ld;
        float* dst = avec + buf * 2 * C;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * lane + h, t = t0 + j;
            const bool ok = t < N;
            cp_async4(dst + j, ok ? al + t : al, ok ? 4u : 0u);
            cp_async4(dst + C + j, ok ? gl + t : gl, ok ? 4u : 0u);
        }
        cp_async_commit();
    };

    if ((int)blockIdx.x < items) {
        if (tid == 0) issue(blockIdx.x);
        if (warp == 1) stage_vectors(blockIdx.x, 0);
    }

    bool bad = false;
    int it = 0;
    for (int item = blockIdx.x; item < items; item += gridDim.x, ++it) {
        const int chain = item / nch, c = item % nch;
        const int next = item + gridDim.x;
        const uint32_t ph = it & 1;

        // M1: [K;Q] K^T
        if (tid == 0) {
            if (!mbar_wait(full, ph, kErrTmaLoad)) {
                bad = true;
            } else {
                tc_fence_after();
                const uint64_t dkq = sdesc_sw128(smem_u32(sm), 16, 1024);
                const uint32_t id = idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = ((ks / 4) * 2 * TILE + (ks % 4) * 32) >> 4;
                    mma_bf16(tbase + P::T_KQ, dkq + off, dkq + off, id, ks > 0);
                }
                mma_commit(bar1);
                ++commits1;
            }
        }
        // decay / gate vectors of this item; stage the next item's
        if (warp == 1) {
            cp_async_wait_all();
            const float* av = avec + (it & 1) * 2 * C;
            const int t = c * C + 2 * lane;
            float La, Lb, Lc;
            chunk_logdecay(av[2 * lane], av[2 * lane + 1], t < N, t + 1 < N, lane, La, Lb, Lc);
            Lv[2 * lane] = La;
            Lv[2 * lane + 1] = Lb;
            bv[2 * lane] = __expf(La);
            bv[2 * lane + 1] = __expf(Lb);
            gv[2 * lane] = av[C + 2 * lane];
            gv[2 * lane + 1] = av[C + 2 * lane + 1];
            // e^{L_t - L_j} = e^{L_t - L_m} e^{L_m - L_j} while both factors stay finite
            const float Lm = __shfl_sync(0xffffffffu, Lb, C / 4 - 1);
            float lo = fminf(La, Lb), hi = fmaxf(La, Lb);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
                hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
            }
            ef[2 * lane] = __expf(La - Lm);
            ef[2 * lane + 1] = __expf(Lb - Lm);
            eg[2 * lane] = __expf(Lm - La);
            eg[2 * lane + 1] = __expf(Lm - Lb);
            if (lane == 0) *factored = (hi - Lm <= 80.f && Lm - lo <= 80.f) ? 1 : 0;
            // the chain pass's per-token factors: b_t, then b_C / b_t
            float* vg = vec + (size_t)item * 2 * C;
            reinterpret_cast<float2*>(vg)[lane] = make_float2(__expf(La), __expf(Lb));
            reinterpret_cast<float2*>(vg + C)[lane] = make_float2(__expf(Lc - La), __expf(Lc - Lb));
            __syncwarp();
            if (next < items) stage_vectors(next, (it + 1) & 1);
        }
        __syncthreads();

        // Kb = diag(b) K into the B operand of M2 (raw K is still read by M1)
        for (int e = tid; e < NB * 8 * C; e += kThreads) {
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            float f[8];
            unpack8(reinterpret_cast<const uint4*>(sm + (2 * b) * TILE)[rem], f);
            reinterpret_cast<uint4*>(kbt + b * TILE)[rem] = pack8(f, bv[row]);
        }

        // score blocks -> A (fp32, strictly lower, gated and decayed) and P~ (bf16)
        if (!mbar_wait(bar1, ph, kErrMma)) bad = true;
        tc_fence_after();
        {
            const int r = acc_row<128>(quad, lane);
            float v[32];
            tmem_ld16(tmem_addr(tbase, quad, P::T_KQ + wg * 32), *reinterpret_cast<float(*)[16]>(v));
            tmem_ld16(tmem_addr(tbase, quad, P::T_KQ + wg * 32 + 16), *reinterpret_cast<float(*)[16]>(v + 16));
            tmem_ld_wait();
            tmem_regs_after_wait(v);
            const bool fact = *factored != 0;
            if (r < 64) {
                const float gr = gv[r], Lr = Lv[r], sr = gr * ef[r];
                if (fact) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int j = wg * 32 + x;
                        As[r * (C + 1) + j] = j < r ? sr * eg[j] * v[x] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 32; ++x) {
                        const int j = wg * 32 + x;
                        As[r * (C + 1) + j] = j < r ? gr * __expf(Lr - Lv[j]) * v[x] : 0.f;
                    }
                }
            } else {
                const int i = r - 64;
                const float Li = Lv[i], si = ef[i];
                uint32_t pk[16];
                if (fact) {
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const int j = wg * 32 + 2 * h;
                        const float a = j <= i ? si * eg[j] * v[2 * h] : 0.f;
                        const float b = j + 1 <= i ? si * eg[j + 1] * v[2 * h + 1] : 0.f;
                        pk[h] = pack_bf16x2(a, b);
                    }
                } else {
#pragma unroll
                    for (int h = 0; h < 16; ++h) {
                        const int j = wg * 32 + 2 * h;
                        const float a = j <= i ? __expf(Li - Lv[j]) * v[2 * h] : 0.f;
                        const float b = j + 1 <= i ? __expf(Li - Lv[j + 1]) * v[2 * h + 1] : 0.f;
                        pk[h] = pack_bf16x2(a, b);
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    *reinterpret_cast<uint4*>(ptile + sw128_offset(i, wg * 64 + q * 16)) =
                        make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
        // M1 has read the K / Q tiles and Kb is built: they take the next item
        if (tid == 0 && next < items) issue(next);

        // T = (I + A)^{-1}: diagonal 16 x 16 blocks (one thread per column) ...
        constexpr int TSt = P::TS;
        if (tid < 64) {
            const int a = tid / 16, l = tid % 16;
            float x[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float sacc = 0.f;
#pragma unroll
                for (int j = 0; j < i; ++j) sacc = fmaf(As[(16 * a + i) * (C + 1) + 16 * a + j], x[j], sacc);
                x[i] = (i == l ? 1.f : 0.f) - sacc;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) Tm[(16 * a + i) * TSt + 16 * a + l] = x[i];
        }
        __syncthreads();
        // ... then block diagonals k = 1..3: X_ab = sum_{c=b}^{a-1} A_ac T_cb and
        // T_ab = -T_aa X_ab, as tf32 warp MMAs; warp w takes pair b = w / 2 of the
        // level and the 8 columns (w % 2) of its block.
        {
            const int g = lane >> 2, t4 = lane & 3;
            float* Xw = Xs + warp * 16 * 9;
#pragma unroll
            for (int k = 1; k <= 3; ++k) {
                if (warp < 2 * (4 - k)) {
                    const int b = warp >> 1, a = b + k, n0 = 16 * b + 8 * (warp & 1);
                    float x[4] = {0.f, 0.f, 0.f, 0.f};
                    for (int kc = 16 * b; kc < 16 * a; kc += 8) {
                        const float* Ap = As + (16 * a) * (C + 1) + kc;
                        const uint32_t af[4] = {to_tf32(Ap[g * (C + 1) + t4]), to_tf32(Ap[(g + 8) * (C + 1) + t4]),
                                                to_tf32(Ap[g * (C + 1) + t4 + 4]),
                                                to_tf32(Ap[(g + 8) * (C + 1) + t4 + 4])};
                        const float* Bp = Tm + kc * TSt + n0;
                        mma_16x8x8_tf32(x, af, to_tf32(Bp[t4 * TSt + g]), to_tf32(Bp[(t4 + 4) * TSt + g]));
                    }
                    Xw[g * 9 + 2 * t4] = x[0];
                    Xw[g * 9 + 2 * t4 + 1] = x[1];
                    Xw[(g + 8) * 9 + 2 * t4] = x[2];
                    Xw[(g + 8) * 9 + 2 * t4 + 1] = x[3];
                    __syncwarp();
                    float y[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int kk = 0; kk < 16; kk += 8) {
                        const float* Ap = Tm + (16 * a) * TSt + 16 * a + kk;
                        const uint32_t af[4] = {to_tf32(Ap[g * TSt + t4]), to_tf32(Ap[(g + 8) * TSt + t4]),
                                                to_tf32(Ap[g * TSt + t4 + 4]), to_tf32(Ap[(g + 8) * TSt + t4 + 4])};
                        mma_16x8x8_tf32(y, af, to_tf32(Xw[(kk + t4) * 9 + g]), to_tf32(Xw[(kk + t4 + 4) * 9 + g]));
                    }
                    float* Dp = Tm + (16 * a) * TSt + n0;
                    Dp[g * TSt + 2 * t4] = -y[0];
                    Dp[g * TSt + 2 * t4 + 1] = -y[1];
                    Dp[(g + 8) * TSt + 2 * t4] = -y[2];
                    Dp[(g + 8) * TSt + 2 * t4 + 1] = -y[3];
                    __syncwarp();
                }
                __syncthreads();
            }
        }
        // T' = T diag(g), bf16, K-major A operand of M2 (T is unit lower triangular)
        for (int e = tid; e < C * 8; e += kThreads) {
            const int i = e / 8, cc = e % 8;
            const float4 t0 = *reinterpret_cast<const float4*>(&Tm[i * TSt + cc * 8]);
            const float4 t1 = *reinterpret_cast<const float4*>(&Tm[i * TSt + cc * 8 + 4]);
            const float tv[8] = {t0.x, t0.y, t0.z, t0.w, t1.x, t1.y, t1.z, t1.w};
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int j = cc * 8 + 2 * h;
                const float a = j <= i ? tv[2 * h] * gv[j] : 0.f;
                const float b = j + 1 <= i ? tv[2 * h + 1] * gv[j + 1] : 0.f;
                pk[h] = pack_bf16x2(a, b);
            }
            *reinterpret_cast<uint4*>(ttile + sw128_offset(i, cc * 16)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // M2: W = T' Kb;  T' and P~ leave for the workspace meanwhile
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dt = sdesc_sw128(smem_u32(ttile), 16, 1024);
            const uint64_t dkb = sdesc_sw128(smem_u32(kbt), TILE, 1024);
            const uint32_t id = idesc_bf16_f32(64, D, 0, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_W, dt + ((ks * 32) >> 4), dkb + ((ks * 2048) >> 4), id, ks > 0);
            mma_commit(bar2);
            ++commits2;
            tma_store_3d(&tm_t, ttile, 0, c * C, chain);
            tma_store_3d(&tm_p, ptile, 0, c * C, chain);
            tma_store_commit();
        }
        if (!mbar_wait(bar2, ph, kErrMma)) bad = true;
        tc_fence_after();
        // -W -> bf16 staging over A (K-major tiles [tokens][64 features])
        {
            const int i = acc_row<64>(quad, lane);
#pragma unroll
            for (int gg = 0; gg < D / 32; gg += 2) {
                const int col0 = wg * (D / 2) + gg * 16;
                float v[32];
                tmem_ld16(tmem_addr(tbase, quad, P::T_W + col0), *reinterpret_cast<float(*)[16]>(v));
                tmem_ld16(tmem_addr(tbase, quad, P::T_W + col0 + 16), *reinterpret_cast<float(*)[16]>(v + 16));
                tmem_ld_wait();
                tmem_regs_after_wait(v);
                if (i >= 0) {
                    unsigned char* blk = wstage + (col0 / 64) * TILE;
                    const int byte0 = (col0 % 64) * 2;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float* w = v + 8 * q;
                        *reinterpret_cast<uint4*>(blk + sw128_offset(i, byte0 + 16 * q)) =
                            make_uint4(pack_bf16x2(-w[0], -w[1]), pack_bf16x2(-w[2], -w[3]),
                                       pack_bf16x2(-w[4], -w[5]), pack_bf16x2(-w[6], -w[7]));
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
        if (tid == 0) {
            for (int b = 0; b < NB; ++b) tma_store_3d(&tm_w, wstage + b * TILE, b * 64, c * C, chain);
            tma_store_commit();
            tma_store_wait_read();   // staging, T' and P~ are rewritten by the next item
        }
    }
    if (warp == 1) cp_async_wait_all();
    if (tid == 0) {
        tma_store_wait_all();
        if (bad) {
            if (loads_issued > 0) mbar_wait(full, (loads_issued - 1) & 1, kErrTmaLoad);
            if (commits1 > 0) mbar_wait(bar1, (commits1 - 1) & 1, kErrMma);
            if (commits2 > 0) mbar_wait(bar2, (commits2 - 1) & 1, kErrMma);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
    // Launched early behind the previous call's kernels (one sequence after
    // another), this grid reads none of their results, but it completes only
    // after them, so the stream still finishes the calls in order.
    grid_dependency_wait();
}

// ===========================================================================
// gd_chain_kernel
// ===========================================================================

template <int D>
struct ChainPlan {
    static constexpr int STAGES = 2;
    static constexpr int NB = D / 64;
    // stage: K[NB] | -W_0 Q_0 -W_1 Q_1 ... | T' Z P~ | V | b[C] r[C]  (Z: a zero tile,
    // never loaded; b_t = e^{L_t}, r_t = b_C / b_t from the prep pass)
    // [-W_b; Q_b], [T'; Z] and [Z; P~] are M = 128 K-major A operands.
    static constexpr int O_K = 0, O_WQ = NB * TILE, O_T = 3 * NB * TILE;
    static constexpr int O_Z = O_T + TILE, O_P = O_Z + TILE, O_V = O_P + TILE;
    static constexpr int O_VEC = O_V + TILE;
    static constexpr int VEC_BYTES = 2 * C * 4;
    static constexpr int STAGE = O_VEC + 1024;                // stages stay 1024-byte aligned
    static constexpr int LOAD_BYTES = (3 * NB + 3) * TILE + VEC_BYTES;
    static constexpr int OFF_SB = STAGES * STAGE;             // S bf16 [D][64], MN-major B operand
    static constexpr int OFF_U = OFF_SB + NB * TILE;          // U bf16 [C][64] (B of P~ U)
    static constexpr int OFF_UH = OFF_U + TILE;               // diag(b_C / b) U bf16 (B of K^T U)
    static constexpr int OFF_O = OFF_UH + TILE;               // output staging
    static constexpr int OFF_BAR = OFF_O + TILE;
    // full[2] empty[2] uo_full[2] o_full[2] o_read[2] s_full u_ready s_ready ostage_full ostage_empty
    // drain[2]
    static constexpr int NBAR = 17;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    // TMEM columns: the two issuers' partial [U; Q S] accumulators X1, X2 and the
    // P~ U accumulator X3 (two buffers each), and the two partial state updates
    static constexpr uint32_t T_X1 = 0, T_X2 = 128, T_X3 = 256, T_S1 = 384, T_S2 = 448, T_COLS = 512;
    static constexpr int KS_HALF = D / 32;                   // K-steps of [-W; Q] S per issuer
};

constexpr int kConv = 256;                   // converter threads (warps 0-7)
constexpr int kChainThreads = kConv + 96;    // + issuer warps 8 and 10, TMA warp 9

// The chain of one (chain, 64 value columns).  Per chunk c with start state S:
//   issuers   X1 = [T'; 0] V (one chunk ahead) + [-W; Q]_1 S_1,  X2 = [-W; Q]_2 S_2
//             (feature halves), so rows 0-63 of X1 + X2 are U and rows 64-127 are Q S;
//             after U is in place: S1 = K_1^T U^, S2 = K_2^T U^ (token halves),
//             U^ = diag(b_C / b) U; then X3 = [0; P~] U.
//   converters  U, U^ to bf16;  S <- b_C S + S1 + S2 (fp32, held in registers), its
//             bf16 copy for the next chunk;  o = diag(b) Q S + P~ U -> staging.
// The converters signal with one arrival per warp.
template <int D>
__global__ void __launch_bounds__(kChainThreads, 1)
gd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_p,
                const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ vec,
                const float* __restrict__ S0, float* __restrict__ S_out, int N, int dv)
{
    using P = ChainPlan<D>;
    constexpr int NB = P::NB;
    grid_launch_dependents();   // a following call's prep pass may start on the idle SMs
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* sbt = sm + P::OFF_SB;
    unsigned char* utile = sm + P::OFF_U;
    unsigned char* uhat = sm + P::OFF_UH;
    unsigned char* ostage = sm + P::OFF_O;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* full = bars;          // TMA -> everyone, per stage
    uint64_t* empty = bars + 2;     // both issuers (commit) -> TMA, per stage
    uint64_t* uo_full = bars + 4;   // both issuers: [U; Q S] partials complete, per TMEM buffer
    uint64_t* o_full = bars + 6;    // issuer B: P~ U complete, per TMEM buffer
    uint64_t* o_read = bars + 8;    // output warps: the buffer's output rows read
    uint64_t* s_full = bars + 10;   // both issuers: state update partials complete
    uint64_t* u_ready = bars + 11;  // U warps: U and U^ in place
    uint64_t* s_ready = bars + 12;  // every converter warp: bf16 state written
    uint64_t* os_full = bars + 13;  // output warps: output staging written
    uint64_t* os_empty = bars + 14; // TMA: output staging read by its store
    uint64_t* drain = bars + 15;    // [2] issuers: every MMA each issued is complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = (warp >> 2) & 1;
    const int ntile = dv / DVT;
    const int chain = blockIdx.x / ntile, j0 = (blockIdx.x % ntile) * DVT;
    const int nch = (N + C - 1) / C;

    if (tid == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 2);
            mbar_init(&uo_full[s], 2);
            mbar_init(&o_full[s], 1);
            mbar_init(&o_read[s], 4);
            mbar_init(&drain[s], 1);
        }
        mbar_init(s_full, 2);
        mbar_init(u_ready, 4);
        mbar_init(s_ready, 8);
        mbar_init(os_full, 4);
        mbar_init(os_empty, 1);
        fence_mbar_init();
    }
    // zero tiles of both stages (rows 64-127 of [T'; Z], rows 0-63 of [Z; P~])
    for (int s = 0; s < P::STAGES; ++s)
        for (int e = tid; e < TILE / 16; e += kChainThreads)
            reinterpret_cast<uint4*>(sm + s * P::STAGE + P::O_Z)[e] = make_uint4(0u, 0u, 0u, 0u);
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    grid_dependency_wait();   // the prep pass's operands are complete

    if (warp == 9) {
        // ---------------- TMA: stage loads and output stores ----------------
        if (lane == 0) {
            const uint64_t pol_once = policy_evict_first();
            const uint64_t pol_shared = ntile > 1 ? policy_evict_normal() : policy_evict_first();
            const float* vchain = vec + (size_t)chain * nch * 2 * C;
            int loads = 0;
            auto issue = [&](int c) {
                const int s = c % P::STAGES;
                unsigned char* st = sm + s * P::STAGE;
                const int y = c * C;
                mbar_expect_tx(&full[s], P::LOAD_BYTES);
                for (int b = 0; b < NB; ++b) {
                    tma_load_3d(st + P::O_K + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol_shared);
                    tma_load_3d(st + P::O_WQ + (2 * b) * TILE, &tm_w, b * 64, y, chain, &full[s], pol_shared);
                    tma_load_3d(st + P::O_WQ + (2 * b + 1) * TILE, &tm_q, b * 64, y, chain, &full[s], pol_shared);
                }
                tma_load_3d(st + P::O_T, &tm_t, 0, y, chain, &full[s], pol_shared);
                tma_load_3d(st + P::O_P, &tm_p, 0, y, chain, &full[s], pol_shared);
                tma_load_3d(st + P::O_V, &tm_v, j0, y, chain, &full[s], pol_once);
                bulk_load(st + P::O_VEC, vchain + (size_t)c * 2 * C, P::VEC_BYTES, &full[s]);
                loads = c + 1;
            };
            // two stages give a load about one chunk of lead time; pulling the
            // operands of the chunk two further ahead into L2 hides the rest
            auto prefetch = [&](int c) {
                const int y = c * C;
                for (int b = 0; b < NB; ++b) {
                    tma_prefetch_3d(&tm_k, b * 64, y, chain);
                    tma_prefetch_3d(&tm_w, b * 64, y, chain);
                    tma_prefetch_3d(&tm_q, b * 64, y, chain);
                }
                tma_prefetch_3d(&tm_t, 0, y, chain);
                tma_prefetch_3d(&tm_p, 0, y, chain);
                tma_prefetch_3d(&tm_v, j0, y, chain);
            };
            auto store = [&](int c) {
                tma_store_3d(&tm_o, ostage, j0, c * C, chain);
                tma_store_commit();
                tma_store_wait_read();
                mbar_arrive(os_empty);
            };
            for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
            for (int c = P::STAGES; c < min(nch, 2 * P::STAGES); ++c) prefetch(c);
            bool ok = true;
            for (int c = 0; c < nch && ok; ++c) {
                if (c >= 1) {
                    ok = mbar_wait(os_full, (c - 1) & 1, kErrMma);
                    if (!ok) break;
                    store(c - 1);
                }
                if (c + P::STAGES < nch) {
                    ok = mbar_wait(&empty[c % P::STAGES], (c / P::STAGES) & 1, kErrMma);
                    if (ok) issue(c + P::STAGES);
                    if (ok && c + 2 * P::STAGES < nch) prefetch(c + 2 * P::STAGES);
                }
            }
            if (ok && mbar_wait(os_full, (nch - 1) & 1, kErrMma)) store(nch - 1);
            tma_store_wait_all();
            // loads in flight must land before the block exits
            for (int c = max(0, loads - P::STAGES); c < loads; ++c)
                mbar_wait(&full[c % P::STAGES], (c / P::STAGES) & 1, kErrTmaLoad);
        }
        __syncwarp();
    } else if (warp == 8 || warp == 10) {
        // ---------------- MMA issuers ----------------
        if (lane == 0) {
            const bool A = warp == 8;
            const uint32_t id = idesc_bf16_f32(128, 64, 0, 1);
            const uint32_t ids = idesc_bf16_f32(D, 64, 1, 1);
            const uint64_t ds = sdesc_sw128(smem_u32(sbt), TILE, 1024);
            const uint64_t du = sdesc_sw128(smem_u32(utile), TILE, 1024);
            const uint64_t duh = sdesc_sw128(smem_u32(uhat), TILE, 1024);
            const uint32_t tx = tbase + (A ? P::T_X1 : P::T_X2);
            const uint32_t tsp = tbase + (A ? P::T_S1 : P::T_S2);
            auto ready = [&](int c) {   // stage c loaded and TMEM buffer c & 1 read out
                if (!mbar_wait(&full[c % P::STAGES], (c / P::STAGES) & 1, kErrTmaLoad)) return false;
                if (c >= 2 && !mbar_wait(&o_read[c & 1], ((c - 2) / 2) & 1, kErrMma)) return false;
                return true;
            };
            auto m0 = [&](int c) {
                if (!ready(c)) return false;
                tc_fence_after();
                unsigned char* st = sm + (c % P::STAGES) * P::STAGE;
                const uint64_t dt = sdesc_sw128(smem_u32(st + P::O_T), 16, 1024);
                const uint64_t dvv = sdesc_sw128(smem_u32(st + P::O_V), TILE, 1024);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tx + (c & 1) * 64, dt + ((ks * 32) >> 4), dvv + ((ks * 2048) >> 4), id, ks > 0);
                return true;
            };
            bool ok = A ? m0(0) : true;
            for (int c = 0; c < nch && ok; ++c) {
                const int s = c % P::STAGES;
                const uint32_t cp = c & 1;
                unsigned char* st = sm + s * P::STAGE;
                const uint32_t txc = tx + cp * 64;
                if (!A && !(ok = ready(c))) break;
                if (!(ok = mbar_wait(s_ready, c & 1, kErrMma))) break;
                tc_fence_after();
                const uint64_t dwq = sdesc_sw128(smem_u32(st + P::O_WQ), 16, 1024);
                const int k0 = A ? 0 : P::KS_HALF;
#pragma unroll
                for (int kk = 0; kk < P::KS_HALF; ++kk) {
                    const int ks = k0 + kk;
                    mma_bf16(txc, dwq + (((ks / 4) * 2 * TILE + (ks % 4) * 32) >> 4), ds + ((ks * 2048) >> 4), id,
                             (A || kk > 0) ? 1u : 0u);
                }
                mma_commit(&uo_full[cp]);
                if (!(ok = mbar_wait(u_ready, c & 1, kErrMma))) break;
                tc_fence_after();
                const uint64_t dk = sdesc_sw128(smem_u32(st + P::O_K), TILE, 1024);
                const int t0 = A ? 0 : 2;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    const int ks = t0 + kk;
                    mma_bf16(tsp, dk + ((ks * 2048) >> 4), duh + ((ks * 2048) >> 4), ids, kk > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
                if (A) {
                    mma_commit(&empty[s]);
                    if (c + 1 < nch) ok = m0(c + 1);
                } else {
                    const uint64_t dzp = sdesc_sw128(smem_u32(st + P::O_Z), 16, 1024);
                    const uint32_t t3 = tbase + P::T_X3 + cp * 64;
#pragma unroll
                    for (int ks = 0; ks < C / 16; ++ks)
                        mma_bf16(t3, dzp + ((ks * 32) >> 4), du + ((ks * 2048) >> 4), id, ks > 0 ? 1u : 0u);
                    mma_commit(&o_full[cp]);
                    mma_commit(&empty[s]);
                }
            }
            // every MMA issued must complete before TMEM is released
            mma_commit(&drain[A ? 0 : 1]);
            mbar_wait(&drain[A ? 0 : 1], 0, kErrMma);
        }
        __syncwarp();
    } else {
        // ---------------- converters (warps 0-7) ----------------
        // Thread (quad, lane) owns row r = 32 quad + lane of the M = 128
        // accumulators, a token of U (quads 0, 1) or of the output (quads 2, 3),
        // and row f of the M = D state accumulators (f = r for D = 128); warpgroup
        // wg owns 32 of the tile's 64 value columns.
        const int r = quad * 32 + lane;
        const int f = acc_row<D>(quad, lane);   // state row (feature) of this thread, or -1
        bool bad = false;
        auto ld32 = [&](uint32_t col, float (&v)[32]) {
            tmem_ld16(tmem_addr(tbase, quad, col), *reinterpret_cast<float(*)[16]>(v));
            tmem_ld16(tmem_addr(tbase, quad, col + 16), *reinterpret_cast<float(*)[16]>(v + 16));
        };
        auto store_row = [&](unsigned char* tile, int row, const float (&v)[32], float w) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                *reinterpret_cast<uint4*>(tile + sw128_offset(row, wg * 64 + q * 16)) =
                    make_uint4(pack_bf16x2(w * v[8 * q], w * v[8 * q + 1]), pack_bf16x2(w * v[8 * q + 2], w * v[8 * q + 3]),
                               pack_bf16x2(w * v[8 * q + 4], w * v[8 * q + 5]),
                               pack_bf16x2(w * v[8 * q + 6], w * v[8 * q + 7]));
        };
        // per-chunk factors of this thread, read from the stage before this warp's
        // arrival that lets the stage be refilled: b_C, and b_t (output rows) or
        // b_C / b_t (U rows) of token r % 64
        float bc = 1.f, tokf = 1.f, tokf_prev = 1.f;
        auto read_factors = [&](int c) {
            if (!mbar_wait(&full[c % P::STAGES], (c / P::STAGES) & 1, kErrTmaLoad)) bad = true;
            const float* vv = reinterpret_cast<const float*>(sm + (c % P::STAGES) * P::STAGE + P::O_VEC);
            bc = vv[C - 1];
            tokf = quad < 2 ? vv[C + r] : vv[r - 64];
        };
        // output rows of chunk cc (accumulator rows 64-127) -> staging
        auto output_tile = [&](int cc, float bt) {
            if (!mbar_wait(&o_full[cc & 1], (cc / 2) & 1, kErrMma)) bad = true;
            if (cc >= 1 && !mbar_wait(os_empty, (cc - 1) & 1, kErrMma)) bad = true;
            tc_fence_after();
            float o[32], w[32];
            const uint32_t col = (cc & 1) * 64 + wg * 32;
            ld32(P::T_X1 + col, o);
            ld32(P::T_X2 + col, w);
            tmem_ld_wait();
            tmem_regs_after_wait(o);
            tmem_regs_after_wait(w);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] += w[x];
            ld32(P::T_X3 + col, w);
            tmem_ld_wait();
            tmem_regs_after_wait(w);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_read[cc & 1]);
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = fmaf(bt, o[x], w[x]);
            store_row(ostage, r - 64, o, 1.f);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(os_full);
        };

        // start state slice S[:, j0:j0+64] in registers and, as bf16, in the B operand
        float sreg[32];
        {
            const float* src = (S0 && f >= 0) ? S0 + ((size_t)chain * D + f) * dv + j0 + wg * 32 : nullptr;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const float4 t = src ? reinterpret_cast<const float4*>(src)[q] : make_float4(0.f, 0.f, 0.f, 0.f);
                sreg[4 * q] = t.x; sreg[4 * q + 1] = t.y; sreg[4 * q + 2] = t.z; sreg[4 * q + 3] = t.w;
            }
            if (f >= 0) store_row(sbt, f, sreg, 1.f);
            read_factors(0);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_ready);
        }

        for (int c = 0; c < nch && !bad; ++c) {
            const uint32_t cp = c & 1;
            if (quad < 2) {
                // U (rows 0-63) -> bf16: U for P~ U, diag(b_C / b) U for the state update
                if (!mbar_wait(&uo_full[cp], (c / 2) & 1, kErrMma)) bad = true;
                tc_fence_after();
                float u[32], w[32];
                ld32(P::T_X1 + cp * 64 + wg * 32, u);
                ld32(P::T_X2 + cp * 64 + wg * 32, w);
                tmem_ld_wait();
                tmem_regs_after_wait(u);
                tmem_regs_after_wait(w);
#pragma unroll
                for (int x = 0; x < 32; ++x) u[x] += w[x];
                store_row(utile, r, u, 1.f);
                store_row(uhat, r, u, tokf);
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(u_ready);
            } else if (c >= 1) {
                output_tile(c - 1, tokf_prev);
            }

            // state S <- b_C S + S1 + S2; its bf16 copy for the next chunk
            if (!mbar_wait(s_full, c & 1, kErrMma)) bad = true;
            tc_fence_after();
            {
                float a[32], b[32];
                ld32(P::T_S1 + wg * 32, a);
                ld32(P::T_S2 + wg * 32, b);
                tmem_ld_wait();
                tmem_regs_after_wait(a);
                tmem_regs_after_wait(b);
                if (f >= 0) {
#pragma unroll
                    for (int x = 0; x < 32; ++x) sreg[x] = fmaf(bc, sreg[x], a[x] + b[x]);
                }
            }
            if (c + 1 < nch) {
                if (f >= 0) store_row(sbt, f, sreg, 1.f);
                tokf_prev = tokf;
                read_factors(c + 1);
                fence_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_ready);
            } else if (f >= 0 && !bad) {
                // final state slice
                float4* dst = reinterpret_cast<float4*>(S_out + ((size_t)chain * D + f) * dv + j0 + wg * 32);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    dst[q] = make_float4(sreg[4 * q], sreg[4 * q + 1], sreg[4 * q + 2], sreg[4 * q + 3]);
            }
        }
        if (quad >= 2 && !bad) output_tile(nch - 1, tokf);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <int D>
cudaError_t launch_gd(const PrefillArgs& a, int prep_ctas, int mark)
{
    const int chains = a.B * a.H;
    const int nch = (a.N + C - 1) / C;
    const int npad = nch * C;
    // workspace: -W [chains][npad][D], T' and P~ [chains][npad][C] (bf16), then
    // the per-token factors b, b_C / b [chains][nch][2][C] (fp32)
    unsigned char* wneg = static_cast<unsigned char*>(a.workspace);
    unsigned char* tp = wneg + (size_t)chains * npad * D * 2;
    unsigned char* pp = tp + (size_t)chains * npad * C * 2;
    float* vec = reinterpret_cast<float*>(pp + (size_t)chains * npad * C * 2);
    CUtensorMap mq, mk, mv, mo, mw, mt, mp;
    if (!make_map(&mq, a.q, D, a.N, chains, a.ld) || !make_map(&mk, a.k, D, a.N, chains, a.ld) ||
        !make_map(&mv, a.v, a.dv, a.N, chains, a.ld) || !make_map(&mo, a.out, a.dv, a.N, chains, a.ld) ||
        !make_map(&mw, wneg, D, npad, chains, npad) || !make_map(&mt, tp, C, npad, chains, npad) ||
        !make_map(&mp, pp, C, npad, chains, npad))
        return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;

    auto k1 = gd_prep_kernel<D>;
    const int s1 = PrepPlan<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return e;
    // all of L1 as shared memory, so that two prep CTAs fit on an SM
    e = cudaFuncSetAttribute(k1, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    const long long items = (long long)chains * nch;
    const int g1 = (int)std::min<long long>(items, prep_ctas > 0 ? prep_ctas : 2LL * sms);
    // behind an earlier call of the same batch (disjoint workspace), the prep
    // pass starts with programmatic serialization too
    cudaLaunchAttribute pdl1[1];
    pdl1[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl1[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t l1 = {};
    l1.gridDim = dim3(g1);
    l1.blockDim = dim3(kThreads);
    l1.dynamicSmemBytes = s1;
    l1.stream = a.stream;
    l1.attrs = pdl1;
    l1.numAttrs = a.pdl_first ? 1 : 0;
    e = cudaLaunchKernelEx(&l1, k1, mq, mk, mw, mt, mp, a.alpha, a.g, vec, a.N, chains, a.ld);
    if (e != cudaSuccess) return e;
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    stage_mark(mark, a.stream);

    auto k2 = gd_chain_kernel<D>;
    const int s2 = ChainPlan<D>::BYTES;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return e;
    // programmatic serialization: the chain kernel sets up while the prep pass
    // finishes, and waits (griddepcontrol.wait) before reading its operands
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(chains * (a.dv / DVT));
    lc.blockDim = dim3(kChainThreads);
    lc.dynamicSmemBytes = s2;
    lc.stream = a.stream;
    lc.attrs = pdl;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, k2, mq, mk, mv, mw, mt, mp, mo, (const float*)vec, (const float*)a.S0, a.S_out,
                           a.N, a.dv);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(mark + 1, a.stream);
    return cudaSuccess;
}

}  // namespace

// The sequence split of a gated-delta call.  The chain pass runs one CTA per
// (chain, 64 value columns); when that leaves most SMs idle, the sequence is cut
// into parts that run as a pipeline: the prep pass of part i + 1 runs on the
// idle SMs while the chain pass of part i runs, and the chain of part i + 1
// starts from the final state of part i.
GdParts gd_parts(int B, int H, int N, int d, int dv)
{
    (void)d;
    GdParts p;
    p.P = 1;
    p.start[0] = 0;
    p.start[1] = N;
    const long long nch = (N + C - 1) / C;
    const long long ctas = (long long)B * H * (dv / DVT);
    if (N >= 8192 && ctas <= 96) {
        // Part i holds about g^i times part 0's chunks.  Part 0's prep pass runs
        // alone, so a short part 0 exposes little of it; the prep pass of part
        // i + 1 runs on the SMs the chain pass leaves idle, at ~0.84 of the
        // chain's speed per token, so it still ends within the chain pass of
        // part i while parts grow by less than 1 / 0.84.  g = 1.16 measured
        // fastest at 65536 tokens (1.08 to 1.20 tried).
        constexpr double g = 1.16;
        const int P = (int)std::min<long long>(kMaxGdParts, nch / 32);
        double wsum = 0.0, w = 1.0;
        for (int i = 0; i < P; ++i, w *= g) wsum += w;
        long long done = 0;
        w = 1.0;
        for (int i = 0; i < P; ++i, w *= g) {
            p.start[i] = (int)(done * C);
            const long long cnt = i == P - 1 ? nch - done : std::max(1LL, std::llround((double)nch * w / wsum));
            done += cnt;
        }
        p.start[P] = N;
        p.P = P;
    }
    return p;
}

namespace {

// Workspace of one part of n tokens: -W, T', P~ (bf16) and the per-token
// factors (fp32), rounded up to 256 bytes.
size_t gd_part_bytes(long long chains, int n, int d)
{
    const size_t nch = (size_t)((n + C - 1) / C);
    const size_t npad = nch * C;
    const size_t b = (size_t)chains * (npad * (size_t)(d + 2 * C) * 2 + nch * 2 * C * sizeof(float));
    return (b + 255) / 256 * 256;
}

}  // namespace

size_t gd_workspace_bytes(int B, int H, int N, int d, int dv)
{
    const GdParts p = gd_parts(B, H, N, d, dv);
    const long long chains = (long long)B * H;
    size_t total = 0;
    for (int i = 0; i < p.P; ++i) total += gd_part_bytes(chains, p.start[i + 1] - p.start[i], d);
    // two fp32 states that carry the chain from one part to the next
    if (p.P > 1) total += 2 * (size_t)chains * d * dv * sizeof(float);
    return total;
}

cudaError_t launch_prefill_tc_gated_delta(const PrefillArgs& a)
{
    if (!a.workspace || a.workspace_bytes < gd_workspace_bytes(a.B, a.H, a.N, a.d, a.dv))
        return cudaErrorInvalidValue;
    const GdParts parts = gd_parts(a.B, a.H, a.N, a.d, a.dv);
    const long long chains = (long long)a.B * a.H;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    // while a chain pass runs, the next part's prep pass gets the other SMs (two CTAs each)
    const int busy = (int)(chains * (a.dv / DVT));
    const int side_ctas = std::max(2, 2 * (sms - busy));
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    size_t off = 0;
    for (int i = 0; i < parts.P; ++i) off += gd_part_bytes(chains, parts.start[i + 1] - parts.start[i], a.d);
    float* carry[2] = {reinterpret_cast<float*>(ws + off),
                       reinterpret_cast<float*>(ws + off) + (size_t)chains * a.d * a.dv};
    const size_t es = 2;   // bf16 elements
    off = 0;
    for (int i = 0; i < parts.P; ++i) {
        const int t0 = parts.start[i];
        const int n = parts.start[i + 1] - t0;
        PrefillArgs pa = a;
        pa.q = static_cast<const char*>(a.q) + (size_t)t0 * a.d * es;
        pa.k = static_cast<const char*>(a.k) + (size_t)t0 * a.d * es;
        pa.v = static_cast<const char*>(a.v) + (size_t)t0 * a.dv * es;
        pa.out = static_cast<char*>(a.out) + (size_t)t0 * a.dv * es;
        pa.alpha = a.alpha + t0;
        pa.g = a.g + t0;
        pa.N = n;
        pa.S0 = i == 0 ? a.S0 : carry[(i - 1) & 1];
        pa.S_out = i == parts.P - 1 ? a.S_out : carry[i & 1];
        pa.workspace = ws + off;
        pa.workspace_bytes = gd_part_bytes(chains, n, a.d);
        off += pa.workspace_bytes;
        // part 0 keeps the call's stream order; each later part's prep pass
        // starts behind the previous chain pass and runs beside it
        pa.pdl_first = i == 0 ? a.pdl_first : true;
        const int prep_ctas = i == 0 ? 0 : side_ctas;
        const cudaError_t e = a.d == 64 ? launch_gd<64>(pa, prep_ctas, 2 * i) : launch_gd<128>(pa, prep_ctas, 2 * i);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

unsigned int read_and_clear_device_error_gdelta(cudaStream_t stream)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbolAsync(&v, sm100::g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, stream) !=
        cudaSuccess)
        return 0;
    cudaStreamSynchronize(stream);
    if (v) {
        const unsigned int zero = 0;
        cudaMemcpyToSymbolAsync(sm100::g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, stream);
        cudaStreamSynchronize(stream);
    }
    return v;
}

}  // namespace la
