// Tensor-core (tcgen05 + TMEM + TMA) prefill for GLA, the per-key-channel
// gate ("Efficient attention variants" §7.2), with bf16 inputs:
//     S_t = diag(alpha_t) S_{t-1} + k_t v_t^T,   o_t = S_t^T q_t
// (no feature map, no normaliser; alpha [B,H,N,d] fp32 in (0, 1]).
//
// Chunk form (derived here; the pages give the recurrence and the remark that
// chunked kernels pass state between chunks, "Efficient attention variants"
// §8).  In a chunk of C = 64 tokens with start state S, per key channel i let
// B_t = sum_{u<=t} log alpha_u (inclusive, within the chunk), B_C its value
// at the chunk's last token and R = (B_0 + B_C) / 2 its midpoint.  Then
//   S_t  = diag(e^{B_t}) S + sum_{j<=t} diag(e^{B_t - B_j}) k_j v_j^T
//   o_t  = (q_t . e^{B_t})^T S + sum_{j<=t} [(q_t . e^{B_t - R}) . (k_j . e^{R - B_j})] v_j
//   S   <- diag(e^{B_C}) S + (K . e^{B_C - B})^T V
// so with Q^ = Q . e^{B}, K^ = K . e^{B_C - B} (factors <= 1) and
// Q~ = Q^ . e^{-R}, K~ = K^ . e^{R - B_C} (factors <= e^{(B_0 - B_C)/2}):
//   MMA1  P  = Q~ K~^T            P~ = causal mask of P           M=64, N=64, K=d
//   MMA3  O  = Q^ S  (S as bf16)                                  M=64, N=dv, K=d
//   MMA2  O += P~ V                                               M=64, N=dv, K=64
//   MMA4  T  = diag(e^{B_C}) T + K^^T V   (fp32 state in TMEM)    M=d,  N=dv, K=64
// A chunk is in range while every channel's log decay across it stays within
// 160 (so no factor exceeds e^80); log alpha is clamped at -70 per token, so a
// closed gate (alpha -> 0) still fits twice in a chunk.  A wider chunk sets
// the device error word (la_prefill_check reports LA_ERR_UNSUPPORTED).
//
// Across the sequence the same three passes as the kernelized modes run:
// segment summaries (Delta S = sum_t diag(e^{B_L - B_t}) k_t v_t^T and the
// segment's per-channel decay e^{B_L}), a scan into segment start states,
// and the chunk loop of every segment from its start state.
#include <cudaTypedefs.h>

#include <algorithm>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int C = 64;             // tokens per chunk
constexpr int TILE = kTileBytes;  // one 64-row x 128-byte swizzled tile (8 KB)
constexpr float kLogAlphaMin = -70.f;
constexpr float kHalfRangeMax = 80.f;

// log alpha of one token of one channel, clamped; tokens past the chunk's end count as alpha = 1
__device__ __forceinline__ float log_gate(float a, bool valid)
{
    return valid ? fmaxf(__logf(a), kLogAlphaMin) : 0.f;
}

// ---------------------------------------------------------------------------
// Kernel A: segment summaries.  Delta S = sum_t diag(e^{B_L - B_t}) k_t v_t^T
// over the tokens of one segment (B inclusive from the segment start, B_L at
// its last token) and the segment's per-channel decay e^{B_L}.  Chunks run
// from the last to the first, so the weights e^{B_L - B_t} (<= 1) follow from
// a running per-channel suffix sum.
template <int D, int DV>
struct GlaSummaryPlan {
    static constexpr int WORKERS = 512;          // sixteen gate warps
    static constexpr int THREADS = WORKERS + 32; // + the issuing warp
    static constexpr int STAGES = (D + DV > 128) ? 3 : 4;
    static constexpr int KB = C * D * 2, VB = C * DV * 2, AB = C * D * 4;
    static constexpr int LOAD_BYTES = KB + VB;   // + the alpha block of the chunk (bulk copy)
    static constexpr int STAGE = KB + VB + AB;
    static constexpr int TPC = WORKERS / D;      // threads per channel in the suffix scan
    static constexpr int TOK = C / TPC;          // tokens per thread
    static constexpr int OFF_TOT = STAGES * STAGE;               // [TPC][D] part sums
    static constexpr int OFF_CARRY = OFF_TOT + TPC * D * 4;      // [D] log decay after the chunk
    static constexpr int OFF_BAR = OFF_CARRY + D * 4;            // full[S], empty[S], wrdy[S], done
    static constexpr int OFF_TMEM = OFF_BAR + (3 * STAGES + 1) * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    static constexpr uint32_t T_S = 0, T_COLS = DV <= 64 ? 64 : 128;
};

// Roles: warps 0..15 (the gate warps) form each chunk's weights and scale its K
// in place, then signal the chunk's stage barrier; lane 0 of warp 16 issues
// the TMA loads and the MMAs, and refills a stage once its MMA is complete, so
// the gate warps never wait for an issue or a refill.
template <int D, int DV>
__global__ void __launch_bounds__(GlaSummaryPlan<D, DV>::THREADS, 1)
gla_summary_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                   const float* __restrict__ alpha, float* __restrict__ ws, int N, int G, int L, int ld)
{
    using P = GlaSummaryPlan<D, DV>;
    grid_launch_dependents();   // the scan may launch now; it waits for this grid's results
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    float* tot = reinterpret_cast<float*>(sm + P::OFF_TOT);
    float* carry = reinterpret_cast<float*>(sm + P::OFF_CARRY);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    uint64_t* wrdy = empty + P::STAGES;   // gate warps: K^ of the stage's chunk in place
    uint64_t* done = wrdy + P::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const bool issuer = tid == P::WORKERS;
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const uint64_t pol = policy_evict_last();   // the chunk loop reads k, v, alpha again
    const float* achain = alpha + (size_t)chain * ld * D;

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&wrdy[s], P::WORKERS / 32);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    if (tid < D) carry[tid] = 0.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    bool bad = false;
    // chunk slot r processes segment chunk nch - 1 - r
    if (issuer) {
        int loads = 0, commits = 0;
        auto issue = [&](int r) {
            const int c = nch - 1 - r;
            const int s = r % P::STAGES;
            unsigned char* st = sm + s * P::STAGE;
            const int y = t0 + c * C;
            const int n = min(C, t1 - y);
            mbar_expect_tx(&full[s], P::LOAD_BYTES + n * D * 4);
            for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol);
            for (int b = 0; b < DV / 64; ++b) tma_load_3d(st + P::KB + b * TILE, &tm_v, b * 64, y, chain, &full[s], pol);
            bulk_load(st + P::KB + P::VB, achain + (size_t)y * D, n * D * 4, &full[s]);
            loads = r + 1;
        };
        for (int r = 0; r < min(nch, P::STAGES); ++r) issue(r);
        const uint32_t id_s = idesc_bf16_f32(D, DV, 1, 1);
        for (int r = 0; r < nch; ++r) {
            const int s = r % P::STAGES;
            if (!mbar_wait(&wrdy[s], (r / P::STAGES) & 1, kErrMma)) { bad = true; break; }
            tc_fence_after();
            // Delta S += K^^T V   (M = d, N = dv)
            const uint32_t ka = smem_u32(sm + s * P::STAGE), va = ka + P::KB;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_S, sdesc_sw128(ka + ks * 2048, TILE, 1024),
                         sdesc_sw128(va + ks * 2048, TILE, 1024), id_s, (r > 0 || ks > 0));
            mma_commit(&empty[s]);
            if (r == nch - 1) mma_commit(done);
            commits = r + 1;
            // refill the stage chunk slot r - 1 used: its MMA was issued a chunk ago
            if (r >= 1 && r - 1 + P::STAGES < nch) {
                if (!mbar_wait(&empty[(r - 1) % P::STAGES], ((r - 1) / P::STAGES) & 1, kErrMma)) { bad = true; break; }
                issue(r - 1 + P::STAGES);
            }
        }
        if (bad) {
            // leave no copy or MMA in flight before TMEM is released
            for (int cc = max(0, loads - P::STAGES); cc < loads; ++cc)
                mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
            if (commits > 0)
                mbar_wait(&empty[(commits - 1) % P::STAGES], ((commits - 1) / P::STAGES) & 1, kErrMma);
        }
    } else if (tid < P::WORKERS) {
        for (int r = 0; r < nch; ++r) {
            const int c = nch - 1 - r;
            const int s = r % P::STAGES;
            unsigned char* kt = sm + s * P::STAGE;
            float* at = reinterpret_cast<float*>(kt + P::KB + P::VB);
            const int n = min(C, t1 - (t0 + c * C));
            if (!mbar_wait(&full[s], (r / P::STAGES) & 1, kErrTmaLoad)) bad = true;
            // per channel i: weight of token t = e^{carry_i + sum_{t < u < chunk end} log alpha_u}
            // (log alpha replaces alpha in place, then the weight replaces log alpha)
            const int i = tid % D, part = tid / D;
            float sum = 0.f;
#pragma unroll
            for (int x = P::TOK - 1; x >= 0; --x) {
                const int t = part * P::TOK + x;
                const float la = log_gate(at[t * D + i], t < n);
                at[t * D + i] = la;
                sum += la;
            }
            tot[part * D + i] = sum;
            if (named_bar_or(1, P::WORKERS, bad)) { bad = true; break; }
            float after = carry[i];   // log decay of the tokens after this thread's part
            for (int q2 = part + 1; q2 < P::TPC; ++q2) after += tot[q2 * D + i];
#pragma unroll
            for (int x = P::TOK - 1; x >= 0; --x) {
                const int t = part * P::TOK + x;
                const float la = at[t * D + i];
                at[t * D + i] = t < n ? __expf(after) : 0.f;
                after += la;
            }
            named_bar(1, P::WORKERS);
            if (part == 0) carry[i] = after;   // now includes this whole chunk
            // K^ = k . weight (zero past the end of the sequence), in place
            for (int e = tid; e < (D / 8) * C; e += P::WORKERS) {
                const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
                const int f0 = b * 64 + (((rem % 8) ^ (row & 7)) * 8);   // first channel of this 16-byte chunk
                uint4* p = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
                const float4 w0 = *reinterpret_cast<const float4*>(at + row * D + f0);
                const float4 w1 = *reinterpret_cast<const float4*>(at + row * D + f0 + 4);
                const float w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                float f[8];
                unpack8(*p, f);
#pragma unroll
                for (int x = 0; x < 8; ++x) f[x] *= w[x];
                *p = pack8(f, 1.f);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&wrdy[s]);
        }
        if (!bad && !mbar_wait(done, 0, kErrMma)) bad = true;
    }
    // every thread agrees whether the summary is complete before it is read out
    const bool any_bad = __syncthreads_or(bad);
    tc_fence_after();
    float* slot = ws + (size_t)unit * (D * DV + D);
    if (!any_bad && tid < P::WORKERS) {
        const int f = acc_row<D>(quad, lane);
        for (int g = wg; g < DV / 16; g += 4) {
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + g * 16), v);
            tmem_ld_wait();
            tmem_regs_after_wait(v);
            if (f >= 0) {
                float4* dst = reinterpret_cast<float4*>(slot + (size_t)f * DV + g * 16);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
            }
        }
        if (tid < D) slot[D * DV + tid] = __expf(carry[tid]);   // the segment's decay e^{B_L}
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
    grid_dependency_wait();
}

// ---------------------------------------------------------------------------
// Kernel B: scan of segment summaries with a per-row (channel) decay.  In
// place: slot s <- state at the start of segment s; writes the final state.
// Grid (chains, kGlaScanSplit) of kGlaScanThreads threads; each thread takes
// 16-byte pieces of state rows (four values of one row share its decay) with
// eight segments' loads in flight, so the scan holds few SMs and the chunk
// kernel, launched behind it, becomes resident on the others meanwhile.
constexpr int kGlaScanThreads = 1024, kGlaScanSplit = 4;

template <int D, int DV>
__global__ void __launch_bounds__(kGlaScanThreads, 1)
gla_scan_kernel(float* __restrict__ ws, const float* __restrict__ S0, float* __restrict__ S_out, int G)
{
    constexpr int SLOT = D * DV + D, S4 = D * DV / 4, BATCH = 8;
    grid_launch_dependents();   // the chunk kernel may set up and load q, k, v meanwhile
    grid_dependency_wait();     // the segment summaries are complete
    const int chain = blockIdx.x;
    float* base = ws + (size_t)chain * G * SLOT;
    const int per = (S4 + gridDim.y - 1) / gridDim.y;   // 16-byte pieces of this CTA
    const int lo = blockIdx.y * per, hi = min(S4, lo + per);
    for (int e = lo + (int)threadIdx.x; e < hi; e += kGlaScanThreads) {
        const int row = (4 * e) / DV;
        float4 acc = S0 ? reinterpret_cast<const float4*>(S0 + (size_t)chain * D * DV)[e]
                        : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s0 = 0; s0 < G; s0 += BATCH) {
            float4 delta[BATCH];
            float dec[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const float* slot = base + (size_t)(s0 + i) * SLOT;
                delta[i] = s0 + i < G ? reinterpret_cast<const float4*>(slot)[e] : make_float4(0.f, 0.f, 0.f, 0.f);
                dec[i] = s0 + i < G ? slot[D * DV + row] : 0.f;   // the decays are never overwritten
            }
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                if (s0 + i < G) {
                    reinterpret_cast<float4*>(base + (size_t)(s0 + i) * SLOT)[e] = acc;
                    acc.x = fmaf(dec[i], acc.x, delta[i].x);
                    acc.y = fmaf(dec[i], acc.y, delta[i].y);
                    acc.z = fmaf(dec[i], acc.z, delta[i].z);
                    acc.w = fmaf(dec[i], acc.w, delta[i].w);
                }
            }
        }
        reinterpret_cast<float4*>(S_out + (size_t)chain * D * DV)[e] = acc;
    }
}

// ---------------------------------------------------------------------------
// Kernel C: the chunk loop of one (chain, segment) from its start state.
template <int D, int DV>
struct GlaChunkPlan {
    static constexpr bool TWO_PER_SM = D == 64 && DV == 64;
    static constexpr int NW = TWO_PER_SM ? 8 : 16;         // worker warps
    static constexpr int NWT = NW * 32;
    static constexpr int THREADS = NWT + 32;               // + the issuer warp
    static constexpr int STAGES = 2;
    // stage: Q~ tiles | K~ tiles | V tiles | alpha block, later Q^ tiles, K^ tiles
    static constexpr int QB = C * D * 2, KB = C * D * 2, VB = C * DV * 2, AB = C * D * 4;
    static constexpr int LOAD_BYTES = QB + KB + VB;        // + the chunk's alpha bytes
    static constexpr int STAGE = QB + KB + VB + AB;
    static constexpr int TPC = NWT / D;                    // threads per channel in the prefix scan
    static constexpr int TOK = C / TPC;
    static constexpr int SBLK = D * 128;                   // one 64-column block of the bf16 state
    static constexpr int OFF_S = STAGES * STAGE;           // S bf16, DV / 64 blocks of D x 64
    static constexpr int OFF_P = OFF_S + (DV / 64) * SBLK; // P~ bf16 [C][C]
    static constexpr int OFF_O = OFF_P + TILE;             // output staging bf16 [C][DV]
    // tot[TPC][D], b0[D], bc[D], r[D], ebc[2][D], e^R[D], e^{B_C - R}[D], slow-path flag[2]
    static constexpr int OFF_VEC = OFF_O + C * DV * 2;
    static constexpr int OFF_BAR = OFF_VEC + (TPC + 7) * D * 4 + 16;
    static constexpr int NBAR = 2 * STAGES + 10;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    static_assert(!TWO_PER_SM || 2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
    static_assert(AB == QB + KB, "Q^ and K^ replace the alpha block");
    static constexpr uint32_t T_P = 0, T_O = 64, T_T = 64 + DV;
    static constexpr uint32_t T_COLS = (T_T + DV <= 256) ? 256 : 512;
};

template <int D, int DV>
__global__ void __launch_bounds__(GlaChunkPlan<D, DV>::THREADS, GlaChunkPlan<D, DV>::TWO_PER_SM ? 2 : 1)
gla_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                 const float* __restrict__ alpha, const float* __restrict__ ws, int N, int G, int L, int ld)
{
    using P = GlaChunkPlan<D, DV>;
    constexpr int NW = P::NW, NWT = P::NWT, NQ = NW / 4;
    grid_launch_dependents();
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* scp = sm + P::OFF_S;
    unsigned char* ptil = sm + P::OFF_P;
    unsigned char* otil = sm + P::OFF_O;
    float* tot = reinterpret_cast<float*>(sm + P::OFF_VEC);
    float* b0v = tot + P::TPC * D;     // B_0 per channel
    float* bcv = b0v + D;              // B_C per channel
    float* rv = bcv + D;               // midpoint R per channel
    float* ebc = rv + D;               // [2][D] e^{B_C} per chunk parity
    float* erv = ebc + 2 * D;          // e^R per channel
    float* ecr = erv + D;              // e^{B_C - R} per channel
    int* slow = reinterpret_cast<int*>(ecr + D);   // [2] some channel has e^R below the normal range
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    uint64_t* phi_rdy = empty + P::STAGES;   // workers: Q~, K~, Q^, K^ of the chunk in place
    uint64_t* w_rdy = phi_rdy + 1;           // workers: bf16 state written, T rescaled
    uint64_t* t_done = phi_rdy + 2;          // MMA3 + MMA4 complete
    uint64_t* p_full = phi_rdy + 3;          // MMA1 complete
    uint64_t* ptil_rdy = phi_rdy + 4;        // workers: P~ written
    uint64_t* o_full = phi_rdy + 5;          // MMA2 complete
    uint64_t* o_read = phi_rdy + 6;          // workers: O read out
    uint64_t* os_full = phi_rdy + 7;         // workers: output staging written
    uint64_t* os_empty = phi_rdy + 8;        // issuer: staging read by its store
    uint64_t* drain = phi_rdy + 9;           // issuer: every MMA it issued is complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = warp < NW;
    const bool issuer = tid == NWT;
    const int quad = warp & 3, qg = warp >> 2;
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const uint64_t pol_in = policy_evict_first();
    const float* achain = alpha + (size_t)chain * ld * D;

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(phi_rdy, NW);
        mbar_init(w_rdy, NW);
        mbar_init(t_done, 1);
        mbar_init(p_full, 1);
        mbar_init(ptil_rdy, NW);
        mbar_init(o_full, 1);
        mbar_init(o_read, NW);
        mbar_init(os_full, NW);
        mbar_init(os_empty, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    auto chunk_len = [&](int c) { return min(C, t1 - (t0 + c * C)); };

    if (issuer) {
        // ---------------- issuer: TMA and MMA ----------------
        bool bad = false;
        int loads = 0;
        auto issue = [&](int c) {
            const int s = c % P::STAGES;
            unsigned char* st = sm + s * P::STAGE;
            const int y = t0 + c * C;
            mbar_expect_tx(&full[s], P::LOAD_BYTES + chunk_len(c) * D * 4);
            for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_q, b * 64, y, chain, &full[s], pol_in);
            for (int b = 0; b < D / 64; ++b)
                tma_load_3d(st + P::QB + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol_in);
            for (int b = 0; b < DV / 64; ++b)
                tma_load_3d(st + P::QB + P::KB + b * TILE, &tm_v, b * 64, y, chain, &full[s], pol_in);
            bulk_load(st + P::QB + P::KB + P::VB, achain + (size_t)y * D, chunk_len(c) * D * 4, &full[s]);
            loads = c + 1;
        };
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
        const uint32_t id1 = idesc_bf16_f32(64, 64, 0, 0);
        const uint32_t ido = idesc_bf16_f32(64, DV, 0, 1);
        const uint32_t idt = idesc_bf16_f32(D, DV, 1, 1);
        const uint64_t dsb = sdesc_sw128(smem_u32(scp), P::SBLK, 1024);
        const uint64_t dp = sdesc_sw128(smem_u32(ptil), 16, 1024);
        for (int c = 0; c < nch; ++c) {
            const int s = c % P::STAGES;
            const uint32_t cp = c & 1;
            unsigned char* st = sm + s * P::STAGE;
            const uint64_t dq = sdesc_sw128(smem_u32(st), 16, 1024);                        // Q~
            const uint64_t dk = sdesc_sw128(smem_u32(st + P::QB), 16, 1024);                // K~
            const uint64_t dvb = sdesc_sw128(smem_u32(st + P::QB + P::KB), TILE, 1024);     // V
            unsigned char* hat = st + P::QB + P::KB + P::VB;
            const uint64_t dqh = sdesc_sw128(smem_u32(hat), 16, 1024);                      // Q^, K-major
            const uint64_t dkh = sdesc_sw128(smem_u32(hat + P::QB), TILE, 1024);            // K^^T, MN-major
            if (!mbar_wait(phi_rdy, cp, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_P, dq + off, dk + off, id1, ks > 0);
            }
            mma_commit(p_full);
            if (!mbar_wait(w_rdy, cp, kErrMma)) { bad = true; break; }
            if (c >= 1 && !mbar_wait(o_read, (c - 1) & 1, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_O, dqh + off, dsb + ((ks * 2048) >> 4), ido, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_T, dkh + ((ks * 2048) >> 4), dvb + ((ks * 2048) >> 4), idt, 1u);
            mma_commit(t_done);
            if (!mbar_wait(ptil_rdy, cp, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_O, dp + ((ks * 32) >> 4), dvb + ((ks * 2048) >> 4), ido, 1u);
            mma_commit(o_full);
            mma_commit(&empty[s]);
            if (c >= 1) {
                if (!mbar_wait(os_full, (c - 1) & 1, kErrMma)) { bad = true; break; }
                for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (c - 1) * C, chain);
                tma_store_commit();
                tma_store_wait_read();
                mbar_arrive(os_empty);
            }
            if (c + P::STAGES < nch) {
                if (!mbar_wait(&empty[s], (c / P::STAGES) & 1, kErrMma)) { bad = true; break; }
                issue(c + P::STAGES);
            }
        }
        if (!bad && nch > 0 && mbar_wait(os_full, (nch - 1) & 1, kErrMma)) {
            for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (nch - 1) * C, chain);
            tma_store_commit();
        }
        tma_store_wait_all();
        for (int cc = max(0, loads - P::STAGES); cc < loads; ++cc)
            mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
        mma_commit(drain);
        mbar_wait(drain, 0, kErrMma);
    } else if (worker) {
        // ---------------- workers ----------------
        bool bad = false;
        // Gate factors of chunk c, in place.  Returns the workers' joint error flag
        // (every worker reaches the same named barriers, errors or not).
        auto gates = [&](int c) -> bool {
            const int n = chunk_len(c);
            unsigned char* st = sm + (c % P::STAGES) * P::STAGE;
            unsigned char* qt = st;
            unsigned char* kt = st + P::QB;
            float* at = reinterpret_cast<float*>(st + P::QB + P::KB + P::VB);
            if (!bad && !mbar_wait(&full[c % P::STAGES], (c / P::STAGES) & 1, kErrTmaLoad)) bad = true;
            // inclusive per-channel prefix of log alpha over the chunk (B), in place
            const int i = tid % D, part = tid / D;
            float la[P::TOK];
            float sum = 0.f;
#pragma unroll
            for (int x = 0; x < P::TOK; ++x) {
                const int t = part * P::TOK + x;
                la[x] = log_gate(at[t * D + i], t < n);
                sum += la[x];
            }
            tot[part * D + i] = sum;
            if (part == 0) b0v[i] = la[0];
            if (tid == 0) slow[c & 1] = 0;
            if (named_bar_or(1, NWT, bad)) return true;
            float acc = 0.f, bc = 0.f;
            for (int q2 = 0; q2 < P::TPC; ++q2) {
                const float tq = tot[q2 * D + i];
                if (q2 < part) acc += tq;
                bc += tq;
            }
#pragma unroll
            for (int x = 0; x < P::TOK; ++x) {
                acc += la[x];
                at[(part * P::TOK + x) * D + i] = acc;
            }
            if (part == 0) {
                const float R = 0.5f * (b0v[i] + bc);
                bcv[i] = bc;
                rv[i] = R;
                ebc[(c & 1) * D + i] = __expf(bc);
                erv[i] = __expf(R);
                ecr[i] = __expf(bc - R);
                if (R < -80.f) slow[c & 1] = 1;
                if (bc - R < -kHalfRangeMax) atomicCAS(&g_device_error, 0u, (unsigned int)kErrRange);
            }
            if (named_bar_or(1, NWT, bad)) return true;
            // Q^ = q e^{B}, Q~ = q e^{B - R}, K^ = k e^{B_C - B}, K~ = k e^{R - B}.  In range,
            // |B - R| <= 80, so e^{B - R} and e^{R - B} are finite and the other two follow
            // with the per-channel constants e^R and e^{B_C - R}; when some channel's e^R is
            // below the normal range (R < -80) each factor is its own exponential instead
            constexpr int PER = (D / 8) * C / NWT;
            const bool fast = slow[c & 1] == 0;
            uint4 qh[PER], kh[PER];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = tid + u * NWT;
                const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
                const int f0 = b * 64 + (((rem % 8) ^ (row & 7)) * 8);
                uint4* pq = reinterpret_cast<uint4*>(qt + b * TILE) + rem;
                uint4* pk = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
                float fq[8], fk[8], fqt[8], fkt[8];
                unpack8(*pq, fq);
                unpack8(*pk, fk);
                const bool valid = row < n;
                float Bv[8], bcv8[8], rv8[8];
                *reinterpret_cast<float4*>(Bv) = *reinterpret_cast<const float4*>(at + row * D + f0);
                *reinterpret_cast<float4*>(Bv + 4) = *reinterpret_cast<const float4*>(at + row * D + f0 + 4);
                *reinterpret_cast<float4*>(bcv8) = *reinterpret_cast<const float4*>(bcv + f0);
                *reinterpret_cast<float4*>(bcv8 + 4) = *reinterpret_cast<const float4*>(bcv + f0 + 4);
                *reinterpret_cast<float4*>(rv8) = *reinterpret_cast<const float4*>(rv + f0);
                *reinterpret_cast<float4*>(rv8 + 4) = *reinterpret_cast<const float4*>(rv + f0 + 4);
                if (fast) {
                    // e^{B} = e^{B - R} e^R and e^{B_C - B} = e^{R - B} e^{B_C - R}: two exponentials a
                    // (token, channel); every factor is within e^{+-80} and e^R is a normal float
                    float er8[8], ecr8[8];
                    *reinterpret_cast<float4*>(er8) = *reinterpret_cast<const float4*>(erv + f0);
                    *reinterpret_cast<float4*>(er8 + 4) = *reinterpret_cast<const float4*>(erv + f0 + 4);
                    *reinterpret_cast<float4*>(ecr8) = *reinterpret_cast<const float4*>(ecr + f0);
                    *reinterpret_cast<float4*>(ecr8 + 4) = *reinterpret_cast<const float4*>(ecr + f0 + 4);
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float d = Bv[x] - rv8[x];
                        const float E = __expf(d), Ei = __expf(-d);
                        fqt[x] = fq[x] * E;
                        fkt[x] = valid ? fk[x] * Ei : 0.f;
                        fq[x] = (fq[x] * E) * er8[x];
                        fk[x] = valid ? (fk[x] * Ei) * ecr8[x] : 0.f;
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 8; ++x) {
                        const float B = Bv[x], bcx = bcv8[x], R = rv8[x];
                        fqt[x] = fq[x] * __expf(B - R);
                        fkt[x] = valid ? fk[x] * __expf(R - B) : 0.f;
                        fq[x] *= __expf(B);
                        fk[x] = valid ? fk[x] * __expf(bcx - B) : 0.f;
                    }
                }
                *pq = pack8(fqt, 1.f);
                *pk = pack8(fkt, 1.f);
                qh[u] = pack8(fq, 1.f);
                kh[u] = pack8(fk, 1.f);
            }
            if (named_bar_or(1, NWT, bad)) return true;   // every B is read before Q^, K^ overwrite it
            unsigned char* hat = reinterpret_cast<unsigned char*>(at);
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = tid + u * NWT;
                const int b = e / (8 * C), rem = e % (8 * C);
                reinterpret_cast<uint4*>(hat + b * TILE)[rem] = qh[u];
                reinterpret_cast<uint4*>(hat + P::QB + b * TILE)[rem] = kh[u];
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(phi_rdy);
            return false;
        };
        // the segment's start state S (from the scan) is read in chunk 0's state step
        grid_dependency_wait();
        const float* slot = ws + (size_t)unit * (D * DV + D);
        bool stop = nch > 0 ? gates(0) : false;

        const int fr = acc_row<D>(quad, lane);
        const int ir = acc_row<64>(quad, lane);
        for (int c = 0; c < nch && !stop; ++c) {
            const uint32_t cp = c & 1;
            // bf16 state S for MMA3, then T <- diag(e^{B_C}) T for the carry
            if (!bad && c >= 1 && !mbar_wait(t_done, (c - 1) & 1, kErrMma)) bad = true;
            tc_fence_after();
            const float eb = fr >= 0 ? ebc[cp * D + fr] : 0.f;
            for (int g = qg; g < DV / 16; g += NQ) {
                float v[16];
                if (c == 0) {
                    // chunk 0: S straight from the scan's slot (16-byte loads), not via TMEM
                    const float4* src = reinterpret_cast<const float4*>(slot + (size_t)(fr >= 0 ? fr : 0) * DV + g * 16);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float4 t = fr >= 0 ? src[x] : make_float4(0.f, 0.f, 0.f, 0.f);
                        v[4 * x] = t.x;
                        v[4 * x + 1] = t.y;
                        v[4 * x + 2] = t.z;
                        v[4 * x + 3] = t.w;
                    }
                } else {
                    tmem_ld16(tmem_addr(tbase, quad, P::T_T + g * 16), v);
                    tmem_ld_wait();
                    tmem_regs_after_wait(v);
                }
                if (fr >= 0) {
                    unsigned char* blk = scp + (g / 4) * P::SBLK;
                    const int byte0 = (g % 4) * 32;
                    *reinterpret_cast<uint4*>(blk + sw128_offset(fr, byte0)) =
                        make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                                   pack_bf16x2(v[6], v[7]));
                    *reinterpret_cast<uint4*>(blk + sw128_offset(fr, byte0 + 16)) =
                        make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                                   pack_bf16x2(v[14], v[15]));
                }
#pragma unroll
                for (int x = 0; x < 16; ++x) v[x] *= eb;
                tmem_st16(tmem_addr(tbase, quad, P::T_T + g * 16), v);
            }
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(w_rdy);

            // P~ = causal mask of P
            if (!bad && !mbar_wait(p_full, cp, kErrMma)) bad = true;
            tc_fence_after();
            // this warp's rows are quad*16 .. quad*16+15: column groups above quad are
            // zero (not loaded), the one at quad is the diagonal block
            for (int g = qg; g < 4; g += NQ) {
                float v[16];
                if (g <= quad) {
                    tmem_ld16(tmem_addr(tbase, quad, P::T_P + g * 16), v);
                    tmem_ld_wait();
                    tmem_regs_after_wait(v);
                } else {
#pragma unroll
                    for (int x = 0; x < 16; ++x) v[x] = 0.f;
                }
                if (ir >= 0) {
                    uint32_t pk[8];
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const int j = g * 16 + 2 * h;
                        pk[h] = pack_bf16x2(j <= ir ? v[2 * h] : 0.f, j + 1 <= ir ? v[2 * h + 1] : 0.f);
                    }
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(ir, g * 32)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(ir, g * 32 + 16)) =
                        make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ptil_rdy);

            // gate factors of the next chunk
            if (c + 1 < nch && gates(c + 1)) { stop = true; }

            // output rows -> staging
            if (!bad && !mbar_wait(o_full, cp, kErrMma)) bad = true;
            tc_fence_after();
            if (!bad && c >= 1 && !mbar_wait(os_empty, (c - 1) & 1, kErrMma)) bad = true;
            // all of this warp's column groups (at most two) per TMEM wait
            {
                constexpr int NGO = (DV / 16 + NQ - 1) / NQ;
                float v[NGO][16];
#pragma unroll
                for (int i = 0; i < NGO; ++i)
                    if (qg + i * NQ < DV / 16) tmem_ld16(tmem_addr(tbase, quad, P::T_O + (qg + i * NQ) * 16), v[i]);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < NGO; ++i) tmem_regs_after_wait(v[i]);
#pragma unroll
                for (int i = 0; i < NGO; ++i) {
                    const int g = qg + i * NQ;
                    if (g < DV / 16 && ir >= 0) {
                        unsigned char* blk = otil + (g / 4) * TILE;
                        const int byte0 = (g % 4) * 32;
                        const float* o = v[i];
                        *reinterpret_cast<uint4*>(blk + sw128_offset(ir, byte0)) =
                            make_uint4(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]), pack_bf16x2(o[4], o[5]),
                                       pack_bf16x2(o[6], o[7]));
                        *reinterpret_cast<uint4*>(blk + sw128_offset(ir, byte0 + 16)) =
                            make_uint4(pack_bf16x2(o[8], o[9]), pack_bf16x2(o[10], o[11]), pack_bf16x2(o[12], o[13]),
                                       pack_bf16x2(o[14], o[15]));
                    }
                }
            }
            tc_fence_before();
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(o_read);
                mbar_arrive(os_full);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
}

template <int D, int DV>
cudaError_t launch_gla(const PrefillArgs& a, const TcSegments& sg)
{
    const int chains = a.B * a.H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, D, a.N, chains, a.ld) || !make_map(&mk, a.k, D, a.N, chains, a.ld) ||
        !make_map(&mv, a.v, DV, a.N, chains, a.ld) || !make_map(&mo, a.out, DV, a.N, chains, a.ld))
        return cudaErrorInvalidValue;
    float* ws = static_cast<float*>(a.workspace);
    const int units = chains * sg.G;

    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.stream = a.stream;
    lc.attrs = pdl;

    auto ka = gla_summary_kernel<D, DV>;
    const int sa = GlaSummaryPlan<D, DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, sa);
    if (e != cudaSuccess) return e;
    lc.gridDim = dim3(units);
    lc.blockDim = dim3(GlaSummaryPlan<D, DV>::THREADS);
    lc.dynamicSmemBytes = sa;
    lc.numAttrs = a.pdl_first ? 1 : 0;
    e = cudaLaunchKernelEx(&lc, ka, mk, mv, a.alpha, ws, a.N, sg.G, sg.L, a.ld);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(0, a.stream);

    lc.gridDim = dim3(chains, kGlaScanSplit);
    lc.blockDim = dim3(kGlaScanThreads);
    lc.dynamicSmemBytes = 0;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, gla_scan_kernel<D, DV>, ws, a.S0, a.S_out, sg.G);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(1, a.stream);

    auto kc = gla_chunk_kernel<D, DV>;
    const int sc = GlaChunkPlan<D, DV>::BYTES;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, sc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    lc.gridDim = dim3(units);
    lc.blockDim = dim3(GlaChunkPlan<D, DV>::THREADS);
    lc.dynamicSmemBytes = sc;
    e = cudaLaunchKernelEx(&lc, kc, mq, mk, mv, mo, a.alpha, (const float*)ws, a.N, sg.G, sg.L, a.ld);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(2, a.stream);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_prefill_tc_gla(const PrefillArgs& a, const TcSegments& sg)
{
    if (!a.workspace || sg.G <= 0 ||
        a.workspace_bytes < (size_t)a.B * a.H * sg.G * ((size_t)a.d * a.dv + a.d) * sizeof(float))
        return cudaErrorInvalidValue;
#define LA_GLA_TC(D, DV) \
    if (a.d == D && a.dv == DV) return launch_gla<D, DV>(a, sg);
    LA_GLA_TC(64, 64)
    LA_GLA_TC(64, 128)
    LA_GLA_TC(128, 64)
    LA_GLA_TC(128, 128)
#undef LA_GLA_TC
    return cudaErrorInvalidValue;
}

unsigned int read_and_clear_device_error_gla(cudaStream_t stream)
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
