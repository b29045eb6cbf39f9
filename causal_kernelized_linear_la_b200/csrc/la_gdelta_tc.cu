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
// With T = (I + A)^{-1}:
//   W = T diag(g b) K,  U~ = T diag(g) V,  U = U~ - W S
//   O = diag(b) Q S + (Q K^T o R) U,  R_tj = e^{L_t-L_j} [j <= t]
//   S_next = b_C S + (diag(b_C / b) K)^T U
// Substituting back reproduces the token recurrence exactly (up to rounding).
//
// One CTA owns one (chain, 64-wide value tile): the columns of S evolve
// independently under the delta rule, so value tiles need no communication.
// Per chunk, all contractions run on the tensor cores:
//   M1  [K;Q] K^T            M=128, N=64, K=d     (both score blocks at once)
//   M2  T' [diag(b)K | V]    M=64,  N=d+64, K=64  (W and U~ together; T' = T diag(g))
//   M3  -W S  (onto U~),  diag(b)Q S   M=64, N=64, K=d
//   M4  P~ U (onto O),  K~^T U (onto S)           M=64 / M=d, N=64, K=64
// T = (I + A)^{-1} is formed on the CUDA cores in fp32 by blocked forward
// substitution (16 x 16 diagonal blocks, then three off-diagonal levels).
#include <cudaTypedefs.h>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int C = 64;            // tokens per chunk
constexpr int DVT = 64;          // value columns per CTA
constexpr int kThreads = 256;    // two warpgroups
constexpr int TILE = kTileBytes; // 64 rows x 128 bytes

template <int D>
struct GdPlan {
    static constexpr int STAGES = 2;
    static constexpr int NB = D / 64;                      // feature blocks
    // stage: [K_0 Q_0 K_1 Q_1 ...] then [Kb_0 .. Kb_{NB-1} V]
    static constexpr int KQ = 2 * NB * TILE;
    static constexpr int WB = (NB + 1) * TILE;
    static constexpr int STAGE = KQ + WB;
    static constexpr int LOAD_BYTES = (2 * NB + 1) * TILE; // TMA bytes per stage
    static constexpr int OFF_P = STAGES * STAGE;           // P~ bf16 [C][C]
    static constexpr int OFF_T = OFF_P + TILE;             // T' bf16 [C][C]; later the output staging tile
    static constexpr int OFF_U = OFF_T + TILE;             // U bf16 [C][DVT]
    static constexpr int OFF_SB = OFF_U + TILE;            // S bf16 [D][DVT]
    static constexpr int OFF_A = OFF_SB + NB * TILE;       // A fp32 [C][C+1]
    static constexpr int OFF_TM = OFF_A + C * (C + 1) * 4; // T fp32 [C][C+1]
    static constexpr int OFF_X = OFF_TM + C * (C + 1) * 4; // off-diagonal scratch fp32 [3][16][17]
    static constexpr int OFF_VEC = OFF_X + 3 * 16 * 17 * 4;// L[C], b[C], g[C], alpha/g [2][2][C]
    static constexpr int OFF_BAR = OFF_VEC + 7 * C * 4;
    static constexpr int NBAR = STAGES + 4;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    // TMEM columns: score blocks, [W | U~], output, state (S: rows = key feature)
    static constexpr uint32_t T_KQ = 0, T_WU = 64, T_O = 256, T_S = 320, T_COLS = 512;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
gdelta_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
              const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
              const float* __restrict__ alpha, const float* __restrict__ gate, const float* __restrict__ S0,
              float* __restrict__ S_out, int N, int dv)
{
    using P = GdPlan<D>;
    constexpr int NB = P::NB;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* ptile = sm + P::OFF_P;
    unsigned char* ttile = sm + P::OFF_T;
    unsigned char* utile = sm + P::OFF_U;
    unsigned char* sbt = sm + P::OFF_SB;
    float* As = reinterpret_cast<float*>(sm + P::OFF_A);
    float* Tm = reinterpret_cast<float*>(sm + P::OFF_TM);
    float* Xs = reinterpret_cast<float*>(sm + P::OFF_X);
    float* Lv = reinterpret_cast<float*>(sm + P::OFF_VEC);
    float* bv = Lv + C;
    float* gv = Lv + 2 * C;
    float* avec = Lv + 3 * C;   // [2][2][C]: alpha, g of two chunks
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* bar1 = full + P::STAGES;
    uint64_t* bar2 = bar1 + 1;
    uint64_t* bar3 = bar1 + 2;
    uint64_t* bar4 = bar1 + 3;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const int ntile = dv / DVT;
    const int chain = blockIdx.x / ntile, j0 = (blockIdx.x % ntile) * DVT;
    const int nch = (N + C - 1) / C;
    const float* al = alpha + (size_t)chain * N;
    const float* gl = gate + (size_t)chain * N;
    const uint64_t pol = policy_evict_first();

    if (tid == 0) {
        for (int s = 0; s < P::NBAR; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    int loads_issued = 0, commits = 0;
    auto issue = [&](int c) {
        const int s = c % P::STAGES;
        unsigned char* st = sm + s * P::STAGE;
        const int y = c * C;
        mbar_expect_tx(&full[s], P::LOAD_BYTES);
        for (int b = 0; b < NB; ++b) {
            tma_load_3d(st + (2 * b) * TILE, &tm_k, b * 64, y, chain, &full[s], pol);
            tma_load_3d(st + (2 * b + 1) * TILE, &tm_q, b * 64, y, chain, &full[s], pol);
        }
        tma_load_3d(st + P::KQ + NB * TILE, &tm_v, j0, y, chain, &full[s], pol);
        loads_issued = c + 1;
    };
    // alpha, g of chunk c into buffer c & 1 (padding past N: alpha = 1, g = 0)
    auto load_vectors = [&](int c) {
        float* dst = avec + (c & 1) * 2 * C;
        // scalar loads: a chain's rows need not be 8-byte aligned when N is odd
        const int t = c * C + lane;
        dst[lane] = t < N ? al[t] : 1.f;
        dst[lane + 32] = t + 32 < N ? al[t + 32] : 1.f;
        dst[C + lane] = t < N ? gl[t] : 0.f;
        dst[C + lane + 32] = t + 32 < N ? gl[t + 32] : 0.f;
    };

    if (tid == 0)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
    if (warp == 1) load_vectors(0);

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
                uint4 c0 = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                      pack_bf16x2(v[6], v[7]));
                uint4 c1 = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                                      pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
                *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2)) = c0;
                *reinterpret_cast<uint4*>(sbt + sw128_offset(f, col0 * 2 + 16)) = c1;
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
        unsigned char* kq = sm + s * P::STAGE;
        unsigned char* wb = kq + P::KQ;

        if (!mbar_wait(&full[s], (c / P::STAGES) & 1, kErrTmaLoad)) bad = true;
        // M1: [K;Q] K^T
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dkq = sdesc_sw128(smem_u32(kq), 16, 1024);
            const uint32_t id = idesc_bf16_f32(128, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * 2 * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_KQ, dkq + off, dkq + off, id, ks > 0);
            }
            mma_commit(bar1);
            commits = c + 1;
        }
        // decay / gate vectors: L = inclusive cumsum of log alpha, b = e^L
        if (warp == 0) {
            const float* av = avec + cp * 2 * C;
            const float l0 = __logf(av[2 * lane]), l1 = __logf(av[2 * lane + 1]);
            float incl = l0 + l1;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const float t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            const float excl = incl - (l0 + l1);
            const float La = excl + l0, Lb = incl;
            Lv[2 * lane] = La; Lv[2 * lane + 1] = Lb;
            bv[2 * lane] = __expf(La); bv[2 * lane + 1] = __expf(Lb);
            gv[2 * lane] = av[C + 2 * lane]; gv[2 * lane + 1] = av[C + 2 * lane + 1];
        }
        if (warp == 1 && c + 1 < nch) load_vectors(c + 1);
        __syncthreads();

        // Kb = diag(b) K into the B operand of M2 (raw K is still read by M1)
        for (int e = tid; e < NB * 8 * C; e += kThreads) {
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            float f[8];
            unpack8(reinterpret_cast<const uint4*>(kq + (2 * b) * TILE)[rem], f);
            reinterpret_cast<uint4*>(wb + b * TILE)[rem] = pack8(f, bv[row]);
        }

        // score blocks -> A (fp32, strictly lower, gated and decayed) and P~ (bf16)
        if (!mbar_wait(bar1, cp, kErrMma)) bad = true;
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
        // K~ = diag(b_C / b) K and Qb = diag(b) Q, in place (M1 is complete)
        {
            const float Llast = Lv[C - 1];
            for (int e = tid; e < NB * 8 * C; e += kThreads) {
                const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
                uint4* pk = reinterpret_cast<uint4*>(kq + (2 * b) * TILE) + rem;
                uint4* pq = reinterpret_cast<uint4*>(kq + (2 * b + 1) * TILE) + rem;
                float f[8];
                unpack8(*pk, f);
                *pk = pack8(f, __expf(Llast - Lv[row]));
                unpack8(*pq, f);
                *pq = pack8(f, bv[row]);
            }
        }
        __syncthreads();

        // T = (I + A)^{-1}: diagonal 16 x 16 blocks (one thread per column) ...
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
            for (int i = 0; i < 16; ++i) Tm[(16 * a + i) * (C + 1) + 16 * a + l] = x[i];
        }
        __syncthreads();
        // ... then block diagonals k = 1..3: X_ab = sum_{c=b}^{a-1} A_ac T_cb, T_ab = -T_aa X_ab
        for (int k = 1; k <= 3; ++k) {
            const int nblk = 4 - k;
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int b = e / 256, a = b + k, i = (e % 256) / 16, j = e % 16;
                float x = 0.f;
                for (int cb = b; cb < a; ++cb)
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        x = fmaf(As[(16 * a + i) * (C + 1) + 16 * cb + m], Tm[(16 * cb + m) * (C + 1) + 16 * b + j], x);
                Xs[(b * 16 + i) * 17 + j] = x;
            }
            __syncthreads();
            for (int e = tid; e < nblk * 256; e += kThreads) {
                const int b = e / 256, a = b + k, i = (e % 256) / 16, j = e % 16;
                float t = 0.f;
                for (int m = 0; m <= i; ++m)
                    t = fmaf(Tm[(16 * a + i) * (C + 1) + 16 * a + m], Xs[(b * 16 + m) * 17 + j], t);
                Tm[(16 * a + i) * (C + 1) + 16 * b + j] = -t;
            }
            __syncthreads();
        }
        // T' = T diag(g), bf16, K-major A operand of M2
        for (int e = tid; e < C * 8; e += kThreads) {
            const int i = e / 8, cc = e % 8;
            uint32_t pk[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const int j = cc * 8 + 2 * h;
                const float a = j <= i ? Tm[i * (C + 1) + j] * gv[j] : 0.f;
                const float b = j + 1 <= i ? Tm[i * (C + 1) + j + 1] * gv[j + 1] : 0.f;
                pk[h] = pack_bf16x2(a, b);
            }
            *reinterpret_cast<uint4*>(ttile + sw128_offset(i, cc * 16)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // M2: [W | U~] = T' [Kb | V]
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dt = sdesc_sw128(smem_u32(ttile), 16, 1024);
            const uint64_t dwb = sdesc_sw128(smem_u32(wb), TILE, 1024);
            const uint32_t id = idesc_bf16_f32(64, D + 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_WU, dt + ((ks * 32) >> 4), dwb + ((ks * 2048) >> 4), id, ks > 0);
            mma_commit(bar2);
        }
        if (!mbar_wait(bar2, cp, kErrMma)) bad = true;
        tc_fence_after();
        // -W -> bf16 over the Kb blocks (K-major A operand of M3)
        {
            const int i = acc_row<64>(quad, lane);
#pragma unroll
            for (int gg = 0; gg < D / 32; ++gg) {
                const int col0 = wg * (D / 2) + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_WU + col0), v);
                tmem_ld_wait();
                if (i >= 0) {
                    unsigned char* blk = wb + (col0 / 64) * TILE;
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

        // M3: U = U~ - W S (onto the U~ columns), O = diag(b) Q S
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dw = sdesc_sw128(smem_u32(wb), 16, 1024);
            const uint64_t dq = sdesc_sw128(smem_u32(kq) + TILE, 16, 1024);
            const uint64_t ds = sdesc_sw128(smem_u32(sbt), TILE, 1024);
            const uint32_t id = idesc_bf16_f32(64, 64, 0, 1);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t b = ds + ((ks * 2048) >> 4);
                mma_bf16(tbase + P::T_WU + D, dw + (((ks / 4) * TILE + (ks % 4) * 32) >> 4), b, id, 1u);
                mma_bf16(tbase + P::T_O, dq + (((ks / 4) * 2 * TILE + (ks % 4) * 32) >> 4), b, id, ks > 0);
            }
            mma_commit(bar3);
        }
        if (!mbar_wait(bar3, cp, kErrMma)) bad = true;
        tc_fence_after();
        {
            // U -> bf16 (MN-major B operand: rows = tokens, 64 value columns)
            const int i = acc_row<64>(quad, lane);
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col0 = wg * 32 + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_WU + D + col0), v);
                tmem_ld_wait();
                if (i >= 0) {
                    *reinterpret_cast<uint4*>(utile + sw128_offset(i, col0 * 2)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(utile + sw128_offset(i, col0 * 2 + 16)) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                }
            }
            // S *= b_C before M4 accumulates K~^T U onto it
            const float bc = bv[C - 1];
            const int f = acc_row<D>(quad, lane);
            (void)f;
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
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // M4: O += P~ U;  S += K~^T U
        if (tid == 0) {
            tc_fence_after();
            const uint64_t dp = sdesc_sw128(smem_u32(ptile), 16, 1024);
            const uint64_t du = sdesc_sw128(smem_u32(utile), TILE, 1024);
            const uint64_t dk = sdesc_sw128(smem_u32(kq), 2 * TILE, 1024);
            const uint32_t ido = idesc_bf16_f32(64, 64, 0, 1);
            const uint32_t ids = idesc_bf16_f32(D, 64, 1, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t b = du + ((ks * 2048) >> 4);
                mma_bf16(tbase + P::T_O, dp + ((ks * 32) >> 4), b, ido, 1u);
                mma_bf16(tbase + P::T_S, dk + ((ks * 2048) >> 4), b, ids, 1u);
            }
            mma_commit(bar4);
        }
        if (!mbar_wait(bar4, cp, kErrMma)) bad = true;
        tc_fence_after();
        if (tid == 0 && c + P::STAGES < nch) issue(c + P::STAGES);   // this stage is free again
        {
            // outputs -> staging (over T', consumed by M2), next chunk's bf16 S
            const int i = acc_row<64>(quad, lane);
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const int col0 = wg * 32 + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_O + col0), v);
                tmem_ld_wait();
                if (i >= 0) {
                    *reinterpret_cast<uint4*>(ttile + sw128_offset(i, col0 * 2)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(ttile + sw128_offset(i, col0 * 2 + 16)) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                }
            }
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
        if (tid == 0) {
            tma_store_3d(&tm_o, ttile, j0, c * C, chain);
            tma_store_commit();
            tma_store_wait_read();   // T' is rewritten in the next chunk
        }
    }
    // final state slice
    if (!bad) {
        tc_fence_after();
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
    if (tid == 0) {
        tma_store_wait_all();
        if (bad) {
            for (int cc = max(0, loads_issued - P::STAGES); cc < loads_issued; ++cc)
                mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
            if (commits > 0) mbar_wait(bar1, (commits - 1) & 1, kErrMma);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
}

template <int D>
cudaError_t launch_gd(const PrefillArgs& a)
{
    const int chains = a.B * a.H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, D, a.N, chains) || !make_map(&mk, a.k, D, a.N, chains) ||
        !make_map(&mv, a.v, a.dv, a.N, chains) || !make_map(&mo, a.out, a.dv, a.N, chains))
        return cudaErrorInvalidValue;
    auto k = gdelta_kernel<D>;
    const int smem = GdPlan<D>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = chains * (a.dv / DVT);
    k<<<grid, kThreads, smem, a.stream>>>(mq, mk, mv, mo, a.alpha, a.g, a.S0, a.S_out, a.N, a.dv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc_gated_delta(const PrefillArgs& a)
{
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
