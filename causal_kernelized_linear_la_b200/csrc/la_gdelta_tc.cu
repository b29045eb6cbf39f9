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
//   S_next = b_C S + K^T diag(b_C / b) U
// Substituting back reproduces the token recurrence exactly (up to rounding).
//
// Only U and S_next depend on the state, so the work splits in two launches:
//   gd_prep_kernel   every (chain, chunk) in parallel: the score blocks
//                    [K;Q]K^T, A and P~, T = (I + A)^{-1} on the CUDA cores in
//                    fp32 (blocked forward substitution), T', W = T' diag(b) K.
//                    Writes -W, T' and P~ (bf16) to the workspace.
//   gd_chain_kernel  one CTA per (chain, 64 value columns), chunks in order:
//                    U = T' V + (-W) S and Q S, then P~ U and the state update,
//                    all on the tensor cores; the CUDA cores only convert U and
//                    S to bf16 operands, scale S by b_C and write the output.
// The columns of S evolve independently under the delta rule, so value tiles
// need no communication.
#include <algorithm>

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
    static constexpr int OFF_X = OFF_TM + C * TS * 4;       // off-diagonal scratch fp32 [3][16][16]
    static constexpr int OFF_VEC = OFF_X + 3 * 16 * 16 * 4; // L[C], b[C], g[C], staged alpha/g [2][2][C]
    static constexpr int OFF_BAR = OFF_VEC + 7 * C * 4;
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
               const float* __restrict__ gate, int N, int chains)
{
    using P = PrepPlan<D>;
    constexpr int NB = P::NB;
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
        const float* al = alpha + (size_t)ch * N;
        const float* gl = gate + (size_t)ch * N;
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
            if (r < 64) {
                const float gr = gv[r], Lr = Lv[r];
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    const int j = wg * 32 + x;
                    As[r * (C + 1) + j] = j < r ? gr * __expf(Lr - Lv[j]) * v[x] : 0.f;
                }
            } else {
                const int i = r - 64;
                const float Li = Lv[i];
                uint32_t pk[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                    const int j = wg * 32 + 2 * h;
                    const float a = j <= i ? __expf(Li - Lv[j]) * v[2 * h] : 0.f;
                    const float b = j + 1 <= i ? __expf(Li - Lv[j + 1]) * v[2 * h + 1] : 0.f;
                    pk[h] = pack_bf16x2(a, b);
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
        // M1 is complete and Kb built: the K/Q tiles take the next item
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
        // ... then block diagonals k = 1..3: X_ab = sum_{c=b}^{a-1} A_ac T_cb, T_ab = -T_aa X_ab.
        // A thread computes one row and four columns of a block (the A element
        // it loads feeds four FMAs; rows of T are read as 16-byte vectors).
#pragma unroll
        for (int k = 1; k <= 3; ++k) {
            const int nblk = 4 - k;
            const bool active = tid < nblk * 64;
            const int b = tid / 64, a = b + k, i = (tid % 64) / 4, j0 = (tid % 4) * 4;
            if (active) {
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int cc = 0; cc < 3; ++cc) {
                    const int cb = b + cc;
                    if (cc < k) {
#pragma unroll
                        for (int m = 0; m < 16; ++m) {
                            const float av = As[(16 * a + i) * (C + 1) + 16 * cb + m];
                            const float4 tv = *reinterpret_cast<const float4*>(&Tm[(16 * cb + m) * TSt + 16 * b + j0]);
                            x.x = fmaf(av, tv.x, x.x);
                            x.y = fmaf(av, tv.y, x.y);
                            x.z = fmaf(av, tv.z, x.z);
                            x.w = fmaf(av, tv.w, x.w);
                        }
                    }
                }
                *reinterpret_cast<float4*>(&Xs[(b * 16 + i) * 16 + j0]) = x;
            }
            __syncthreads();
            if (active) {
                float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    if (m <= i) {
                        const float tv = Tm[(16 * a + i) * TSt + 16 * a + m];
                        const float4 xv = *reinterpret_cast<const float4*>(&Xs[(b * 16 + m) * 16 + j0]);
                        y.x = fmaf(tv, xv.x, y.x);
                        y.y = fmaf(tv, xv.y, y.y);
                        y.z = fmaf(tv, xv.z, y.z);
                        y.w = fmaf(tv, xv.w, y.w);
                    }
                }
                *reinterpret_cast<float4*>(&Tm[(16 * a + i) * TSt + 16 * b + j0]) =
                    make_float4(-y.x, -y.y, -y.z, -y.w);
            }
            __syncthreads();
        }
        // T' = T diag(g), bf16, K-major A operand of M2 (T is unit lower triangular)
        for (int e = tid; e < C * 8; e += kThreads) {
            const int i = e / 8, cc = e % 8;
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int j = cc * 8 + 2 * h;
                const float a = j <= i ? Tm[i * TSt + j] * gv[j] : 0.f;
                const float b = j + 1 <= i ? Tm[i * TSt + j + 1] * gv[j + 1] : 0.f;
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
            for (int gg = 0; gg < D / 32; ++gg) {
                const int col0 = wg * (D / 2) + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_W + col0), v);
                tmem_ld_wait();
                if (i >= 0) {
                    unsigned char* blk = wstage + (col0 / 64) * TILE;
                    const int byte0 = (col0 % 64) * 2;
                    *reinterpret_cast<uint4*>(blk + sw128_offset(i, byte0)) =
                        make_uint4(pack_bf16x2(-v[0], -v[1]), pack_bf16x2(-v[2], -v[3]), pack_bf16x2(-v[4], -v[5]),
                                   pack_bf16x2(-v[6], -v[7]));
                    *reinterpret_cast<uint4*>(blk + sw128_offset(i, byte0 + 16)) =
                        make_uint4(pack_bf16x2(-v[8], -v[9]), pack_bf16x2(-v[10], -v[11]),
                                   pack_bf16x2(-v[12], -v[13]), pack_bf16x2(-v[14], -v[15]));
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
}

// ===========================================================================
// gd_chain_kernel
// ===========================================================================

template <int D>
struct ChainPlan {
    static constexpr int STAGES = 2;
    static constexpr int NB = D / 64;
    // stage: K[NB] Q[NB] -W[NB] T' P~ V
    static constexpr int O_K = 0, O_Q = NB * TILE, O_W = 2 * NB * TILE, O_T = 3 * NB * TILE;
    static constexpr int O_P = O_T + TILE, O_V = O_P + TILE;
    static constexpr int STAGE = O_V + TILE;                // all of it arrives by TMA
    static constexpr int OFF_SB = STAGES * STAGE;           // S bf16 [D][64], MN-major B operand
    static constexpr int OFF_U = OFF_SB + NB * TILE;        // U bf16 [C][64], MN-major B operand
    static constexpr int OFF_UH = OFF_U + TILE;             // diag(b_C / b) U
    static constexpr int OFF_O = OFF_UH + TILE;             // output staging
    static constexpr int OFF_VEC = OFF_O + TILE;            // b[3][C], r[3][C], staged alpha [2][C]
    static constexpr int OFF_BAR = OFF_VEC + 8 * C * 4;
    static constexpr int NBAR = STAGES + 2;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    // TMEM columns: U, Q S (two buffers), P~ U (two buffers), state (rows = key feature)
    static constexpr uint32_t T_U = 0, T_O1 = 64, T_O2 = 192, T_S = 320, T_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
gd_chain_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_w,
                const __grid_constant__ CUtensorMap tm_t, const __grid_constant__ CUtensorMap tm_p,
                const __grid_constant__ CUtensorMap tm_o, const float* __restrict__ alpha,
                const float* __restrict__ S0, float* __restrict__ S_out, int N, int dv)
{
    using P = ChainPlan<D>;
    constexpr int NB = P::NB;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* sbt = sm + P::OFF_SB;
    unsigned char* utile = sm + P::OFF_U;
    unsigned char* uhtile = sm + P::OFF_UH;
    unsigned char* ostage = sm + P::OFF_O;
    float* vb_b = reinterpret_cast<float*>(sm + P::OFF_VEC);   // [3][C] b_i
    float* vb_r = vb_b + 3 * C;                                // [3][C] b_C / b_i
    float* abuf = vb_b + 6 * C;                                // [2][C] staged alpha
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* bar3 = full + P::STAGES;
    uint64_t* bar4 = bar3 + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const int ntile = dv / DVT;
    const int chain = blockIdx.x / ntile, j0 = (blockIdx.x % ntile) * DVT;
    const int nch = (N + C - 1) / C;
    const float* al = alpha + (size_t)chain * N;
    const uint64_t pol_once = policy_evict_first();
    const uint64_t pol_shared = ntile > 1 ? policy_evict_normal() : policy_evict_first();

    if (tid == 0) {
        for (int s = 0; s < P::NBAR; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    int loads_issued = 0, commits3 = 0, commits4 = 0;
    auto issue = [&](int c) {
        const int s = c % P::STAGES;
        unsigned char* st = sm + s * P::STAGE;
        const int y = c * C;
        mbar_expect_tx(&full[s], P::STAGE);
        for (int b = 0; b < NB; ++b) {
            tma_load_3d(st + P::O_K + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol_shared);
            tma_load_3d(st + P::O_Q + b * TILE, &tm_q, b * 64, y, chain, &full[s], pol_shared);
            tma_load_3d(st + P::O_W + b * TILE, &tm_w, b * 64, y, chain, &full[s], pol_shared);
        }
        tma_load_3d(st + P::O_T, &tm_t, 0, y, chain, &full[s], pol_shared);
        tma_load_3d(st + P::O_P, &tm_p, 0, y, chain, &full[s], pol_shared);
        tma_load_3d(st + P::O_V, &tm_v, j0, y, chain, &full[s], pol_once);
        loads_issued = c + 1;
    };
    // warp 1: alpha of chunk c into staging buffer c & 1
    auto stage_alpha = [&](int c) {
        float* dst = abuf + (c & 1) * C;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = 2 * lane + h, t = c * C + j;
            const bool ok = t < N;
            cp_async4(dst + j, ok ? al + t : al, ok ? 4u : 0u);
        }
        cp_async_commit();
    };
    // warp 1: b_i and b_C / b_i of chunk c into vector buffer c % 3
    auto chunk_vectors = [&](int c) {
        cp_async_wait_all();
        const float* a = abuf + (c & 1) * C;
        const int t = c * C + 2 * lane;
        float La, Lb, Lc;
        chunk_logdecay(a[2 * lane], a[2 * lane + 1], t < N, t + 1 < N, lane, La, Lb, Lc);
        float* b = vb_b + (c % 3) * C;
        float* r = vb_r + (c % 3) * C;
        b[2 * lane] = __expf(La);
        b[2 * lane + 1] = __expf(Lb);
        r[2 * lane] = __expf(Lc - La);
        r[2 * lane + 1] = __expf(Lc - Lb);
        __syncwarp();
    };
    // output rows of chunk cc: o_i = b_i (Q S)_i + (P~ U)_i  -> bf16 staging
    auto output_tile = [&](int cc) {
        const int i = acc_row<64>(quad, lane);
        const float* b = vb_b + (cc % 3) * C;
        const float bi = i >= 0 ? b[i] : 0.f;
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int col0 = wg * 32 + gg * 16;
            float x1[16], x2[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_O1 + (cc & 1) * 64 + col0), x1);
            tmem_ld16(tmem_addr(tbase, quad, P::T_O2 + (cc & 1) * 64 + col0), x2);
            tmem_ld_wait();
            if (i >= 0) {
                float o[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) o[x] = fmaf(bi, x1[x], x2[x]);
                *reinterpret_cast<uint4*>(ostage + sw128_offset(i, col0 * 2)) =
                    make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                               pack_bf16x2(o[6], o[7]));
                *reinterpret_cast<uint4*>(ostage + sw128_offset(i, col0 * 2 + 16)) =
                    make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                               pack_bf16x2(o[14], o[15]));
            }
        }
    };

    if (tid == 0)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
    if (warp == 1) {
        stage_alpha(0);
        chunk_vectors(0);
        if (nch > 1) stage_alpha(1);
    }

    // start state slice S[:, j0:j0+64] into TMEM (rows = key feature) and bf16 smem
    {
        const int f = acc_row<D>(quad, lane);
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int col0 = wg * 32 + gg * 16;
            float v[16];
#pragma unroll
            for (int x = 0; x < 16; ++x)
                v[x] = (f >= 0 && S0) ? S0[((size_t)chain * D + f) * dv + j0 + col0 + x] : 0.f;
            if (f >= 0) {
                *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2)) =
                    make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7]));
                *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2 + 16)) =
                    make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                               pack_bf16x2(v[14], v[15]));
            }
            tmem_st16(tmem_addr(tbase, quad, P::T_S + col0), v);
        }
        tmem_st_wait();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    bool bad = false;
    for (int c = 0; c < nch; ++c) {
        const int s = c % P::STAGES;
        const uint32_t cp = c & 1;
        unsigned char* st = sm + s * P::STAGE;

        // U = T' V + (-W) S;  Q S  (both read the bf16 copy of S)
        if (tid == 0) {
            if (!mbar_wait(&full[s], (c / P::STAGES) & 1, kErrTmaLoad)) {
                bad = true;
            } else {
                tc_fence_after();
                const uint32_t id = idesc_bf16_f32(64, 64, 0, 1);
                const uint64_t dt = sdesc_sw128(smem_u32(st + P::O_T), 16, 1024);
                const uint64_t dvv = sdesc_sw128(smem_u32(st + P::O_V), TILE, 1024);
#pragma unroll
                for (int ks = 0; ks < C / 16; ++ks)
                    mma_bf16(tbase + P::T_U, dt + ((ks * 32) >> 4), dvv + ((ks * 2048) >> 4), id, ks > 0);
                const uint64_t dw = sdesc_sw128(smem_u32(st + P::O_W), 16, 1024);
                const uint64_t dq = sdesc_sw128(smem_u32(st + P::O_Q), 16, 1024);
                const uint64_t ds = sdesc_sw128(smem_u32(sbt), TILE, 1024);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                    const uint64_t b = ds + ((ks * 2048) >> 4);
                    mma_bf16(tbase + P::T_U, dw + off, b, id, 1u);
                    mma_bf16(tbase + P::T_O1 + cp * 64, dq + off, b, id, ks > 0);
                }
                mma_commit(bar3);
                commits3 = c + 1;
            }
        }
        // S *= b_C in TMEM (the MMAs above read only the bf16 copy)
        {
            const float bc = vb_b[(c % 3) * C + C - 1];
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col0 = wg * 32 + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < 16; ++x) v[x] *= bc;
                tmem_st16(tmem_addr(tbase, quad, P::T_S + col0), v);
            }
            tmem_st_wait();
        }
        // output of the previous chunk (its accumulators are complete)
        if (c >= 1) output_tile(c - 1);
        if (warp == 1 && c + 1 < nch) {
            chunk_vectors(c + 1);
            if (c + 2 < nch) stage_alpha(c + 2);
        }

        // U -> bf16 (MN-major B operand) and diag(b_C / b) U
        if (!mbar_wait(bar3, cp, kErrMma)) bad = true;
        tc_fence_after();
        {
            const int i = acc_row<64>(quad, lane);
            const float ri = i >= 0 ? vb_r[(c % 3) * C + i] : 0.f;
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col0 = wg * 32 + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_U + col0), v);
                tmem_ld_wait();
                if (i >= 0) {
                    *reinterpret_cast<uint4*>(utile + sw128_offset(i, col0 * 2)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(utile + sw128_offset(i, col0 * 2 + 16)) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                    *reinterpret_cast<uint4*>(uhtile + sw128_offset(i, col0 * 2)) =
                        make_uint4(pack_bf16x2(ri * v[0], ri * v[1]), pack_bf16x2(ri * v[2], ri * v[3]),
                                   pack_bf16x2(ri * v[4], ri * v[5]), pack_bf16x2(ri * v[6], ri * v[7]));
                    *reinterpret_cast<uint4*>(uhtile + sw128_offset(i, col0 * 2 + 16)) =
                        make_uint4(pack_bf16x2(ri * v[8], ri * v[9]), pack_bf16x2(ri * v[10], ri * v[11]),
                                   pack_bf16x2(ri * v[12], ri * v[13]), pack_bf16x2(ri * v[14], ri * v[15]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // P~ U (onto its own accumulator);  S += K^T diag(b_C / b) U
        if (tid == 0) {
            tc_fence_after();
            if (c >= 1) {
                tma_store_3d(&tm_o, ostage, j0, (c - 1) * C, chain);
                tma_store_commit();
            }
            const uint32_t ido = idesc_bf16_f32(64, 64, 0, 1);
            const uint32_t ids = idesc_bf16_f32(D, 64, 1, 1);
            const uint64_t dp = sdesc_sw128(smem_u32(st + P::O_P), 16, 1024);
            const uint64_t dk = sdesc_sw128(smem_u32(st + P::O_K), TILE, 1024);
            const uint64_t du = sdesc_sw128(smem_u32(utile), TILE, 1024);
            const uint64_t duh = sdesc_sw128(smem_u32(uhtile), TILE, 1024);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                mma_bf16(tbase + P::T_O2 + cp * 64, dp + ((ks * 32) >> 4), du + ((ks * 2048) >> 4), ido, ks > 0);
                mma_bf16(tbase + P::T_S, dk + ((ks * 2048) >> 4), duh + ((ks * 2048) >> 4), ids, 1u);
            }
            mma_commit(bar4);
            commits4 = c + 1;
        }
        if (!mbar_wait(bar4, cp, kErrMma)) bad = true;
        tc_fence_after();
        if (tid == 0) {
            if (c + P::STAGES < nch) issue(c + P::STAGES);   // this stage is free again
            tma_store_wait_read();                           // the staging tile is rewritten next chunk
        }
        // next chunk's bf16 S
        {
            const int f = acc_row<D>(quad, lane);
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col0 = wg * 32 + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
                tmem_ld_wait();
                if (f >= 0) {
                    *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2 + 16)) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
    }
    if (!bad) {
        // last output tile and the final state slice
        output_tile(nch - 1);
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
            tma_store_3d(&tm_o, ostage, j0, (nch - 1) * C, chain);
            tma_store_commit();
        }
        const int f = acc_row<D>(quad, lane);
#pragma unroll
        for (int gg = 0; gg < 2; ++gg) {
            const int col0 = wg * 32 + gg * 16;
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
            tmem_ld_wait();
            if (f >= 0) {
                float4* dst = reinterpret_cast<float4*>(S_out + ((size_t)chain * D + f) * dv + j0 + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
    }
    if (warp == 1) cp_async_wait_all();
    if (tid == 0) {
        tma_store_wait_all();
        if (bad) {
            for (int cc = max(0, loads_issued - P::STAGES); cc < loads_issued; ++cc)
                mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
            if (commits3 > 0) mbar_wait(bar3, (commits3 - 1) & 1, kErrMma);
            if (commits4 > 0) mbar_wait(bar4, (commits4 - 1) & 1, kErrMma);
        }
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
cudaError_t launch_gd(const PrefillArgs& a)
{
    const int chains = a.B * a.H;
    const int nch = (a.N + C - 1) / C;
    const int npad = nch * C;
    unsigned char* ws = static_cast<unsigned char*>(a.workspace);
    unsigned char* wneg = ws;
    unsigned char* tp = wneg + (size_t)chains * npad * D * 2;
    unsigned char* pp = tp + (size_t)chains * npad * C * 2;
    CUtensorMap mq, mk, mv, mo, mw, mt, mp;
    if (!make_map(&mq, a.q, D, a.N, chains) || !make_map(&mk, a.k, D, a.N, chains) ||
        !make_map(&mv, a.v, a.dv, a.N, chains) || !make_map(&mo, a.out, a.dv, a.N, chains) ||
        !make_map(&mw, wneg, D, npad, chains) || !make_map(&mt, tp, C, npad, chains) ||
        !make_map(&mp, pp, C, npad, chains))
        return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;

    auto k1 = gd_prep_kernel<D>;
    const int s1 = PrepPlan<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
    if (e != cudaSuccess) return e;
    const long long items = (long long)chains * nch;
    const int g1 = (int)std::min<long long>(items, 2LL * sms);
    k1<<<g1, kThreads, s1, a.stream>>>(mq, mk, mw, mt, mp, a.alpha, a.g, a.N, chains);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    auto k2 = gd_chain_kernel<D>;
    const int s2 = ChainPlan<D>::BYTES;
    e = cudaFuncSetAttribute(k2, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
    if (e != cudaSuccess) return e;
    k2<<<chains * (a.dv / DVT), kThreads, s2, a.stream>>>(mq, mk, mv, mw, mt, mp, mo, a.alpha, a.S0, a.S_out,
                                                           a.N, a.dv);
    return cudaGetLastError();
}

}  // namespace

size_t gd_workspace_bytes(int B, int H, int N, int d, int dv)
{
    (void)dv;
    const size_t npad = (size_t)((N + C - 1) / C) * C;
    return (size_t)B * H * npad * (size_t)(d + 2 * C) * 2;
}

cudaError_t launch_prefill_tc_gated_delta(const PrefillArgs& a)
{
    if (!a.workspace || a.workspace_bytes < gd_workspace_bytes(a.B, a.H, a.N, a.d, a.dv))
        return cudaErrorInvalidValue;
    if (a.d == 64) return launch_gd<64>(a);
    return launch_gd<128>(a);
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
