// Tensor-core (tcgen05 + TMEM + TMA) prefill for the kernelized modes
// (LA_PLAIN, LA_DECAY) with bf16 inputs.
//
// Method ("What Is Linear Attention?" §4/§5.1; "Efficient attention
// variants" §5, §7.1 and §8 "chunkwise": parallel inside a chunk, state passed
// between chunks).  For a chunk of C = 64 tokens with start state (S, z),
// local positions i, j and lambda = log gamma_h:
//   P~_ij = [j <= i] gamma^(i-j) phi(q_i).phi(k_j)         (bf16, fp32 products)
//   o_i   = (sum_j P~_ij v_j + gamma^(i+1) S^T phi(q_i)) /
//           (sum_j P~_ij     + gamma^(i+1) z.phi(q_i) + eps)
//   S    <- gamma^n S + K~^T V,  z <- gamma^n z + sum_j K~_j,
//   K~_j  = gamma^(n-1-j) phi(k_j)   (n valid tokens in the chunk)
// The causal mask is multiplicative ("Transformers Are RNNs" notes).
//
// The products are laid out so every contraction runs on the tensor cores:
//   MMA1  P    = phi(Q) phi(K)^T      M=C,  N=C,  K=d    (TMEM, M=64 layout)
//   MMA3  O^T  = S^T phi(Q)^T         M=dv, N=C,  K=d    (start-state read)
//   MMA2  O^T += V^T P~^T             M=dv, N=C,  K=C    (intra-chunk)
//   MMA4  S   += K~^T V               M=d,  N=dv, K=C    (state carry, fp32 in TMEM)
// Putting dv (not the 64 tokens) on the M axis keeps the big products at
// M = 128 and the output tile in TMEM with one value column per thread.
//
// Parallelism across the sequence ("Transformers Are RNNs" notes: the state
// is a prefix sum, so it can be scanned): each (chain, segment) of L tokens
// is one CTA.  Kernel A reduces every segment to its summary
// (Delta S, Delta z); kernel B scans summaries into segment start states and
// the final state; kernel C runs the chunk loop of every segment from its
// true start state.
//
// Supported decay range on this path: gamma >= 0.3 (64 |log gamma| <= 80);
// smaller gamma sets the device error word (la_prefill_check reports it).
#include <cudaTypedefs.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int C = 64;             // tokens per chunk
constexpr int kThreads = 512;     // four warpgroups; each phase is split by columns
constexpr int TILE = C * 64 * 2;  // one 64-row x 128-byte swizzled tile (8 KB)
// The scaled-frame exponents (decay) stay within +-kFrameLimit in natural-log
// units, far from the fp32 / bf16 overflow at ~88.
constexpr float kFrameLimit = 40.f;

// ---------------------------------------------------------------------------
// Shared-memory plan of the chunk kernel (all tiles 1024-byte aligned).
template <int D, int DV, bool DECAY>
struct ChunkPlan {
    // d = dv = 64: two CTAs share an SM (three stages, 256 TMEM columns, at
    // most 60 registers a thread), so one CTA's waits hide behind the other's work
    static constexpr bool TWO_PER_SM = D == 64 && DV == 64;
    static constexpr int STAGES = TWO_PER_SM ? (DECAY ? 2 : 3) : (D + DV > 128) ? 3 : 4;
    static constexpr int QB = C * D * 2, KB = C * D * 2, VB = C * DV * 2;
    static constexpr int STAGE = QB + KB + VB;
    static constexpr int OFF_KH = STAGES * STAGE;                 // K^ (frame-weighted phi(K)), decay only
    static constexpr int OFF_Q32 = OFF_KH + (DECAY ? KB : 0);     // Q^ fp32 [C][D], tf32 operand
    static constexpr int OFF_P = OFF_Q32 + C * D * 4;             // P~ bf16 [C][C]
    // The ones-row A operand of the normaliser MMA: only its row 0 (128
    // bytes) must hold ones; rows 1..63 feed accumulator rows that are never
    // read, so they overlap the small vectors below and the staging tile.
    static constexpr int OFF_ONES = OFF_P + C * C * 2;
    static constexpr int OFF_RDEN = OFF_ONES + 128;               // [C] 1 / denominator
    static constexpr int OFF_DTAB = OFF_RDEN + C * 4;             // [C] gamma^k
    static constexpr int OFF_O = OFF_ONES + 1024;                 // output staging bf16 [C][DV]
    static constexpr int OFF_RSP = OFF_O + C * DV * 2;            // [4][C] row sums of P~ per warpgroup
    static constexpr int OFF_DINT = OFF_RSP + 4 * C * 4;          // [2][C] Q^ . z per chunk parity
    static constexpr int OFF_ZS = OFF_DINT + 2 * C * 4;           // [2][D] z at chunk start per parity
    static constexpr int OFF_BAR = OFF_ZS + 2 * D * 4;
    static constexpr int NBAR = STAGES + 5;                       // full[S], p, s, o, pt_full, o_free
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;            // + alignment slack
    static_assert(OFF_DTAB + C * 4 <= OFF_O, "vectors overlap the staging tile");
    static_assert(OFF_ONES + 8 * 1024 <= OFF_RSP, "ones operand must stay inside the plan");
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    // TMEM columns: scores, output^T, state^T, normaliser row
    static constexpr uint32_t T_P = 0, T_O = 64, T_S = 128;
    static constexpr uint32_t T_Z = TWO_PER_SM ? 192 : 256, T_COLS = TWO_PER_SM ? 256 : 512;
    static_assert(!TWO_PER_SM || 2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
};

template <int D, int DV>
struct SummaryPlan {
    static constexpr int STAGES = 4;
    static constexpr int KB = C * D * 2, VB = C * DV * 2;
    // stage: K tiles, V tiles, then a constant tile whose column 0 is ones:
    // B = [V | 1] makes column dv of K~^T B the normaliser sum Delta z
    static constexpr int LOAD_BYTES = KB + VB;
    static constexpr int STAGE = KB + VB + TILE;
    static constexpr int OFF_BAR = STAGES * STAGE;                // full[S], empty[S], done
    static constexpr int OFF_TMEM = OFF_BAR + (2 * STAGES + 1) * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static constexpr int NS = DV + 16;                            // accumulator columns
    static constexpr uint32_t T_S = 0, T_COLS = 256;
};


// ---------------------------------------------------------------------------
// Kernel A: segment summaries  Delta S = sum_t gamma^(last-t) phi(k_t) v_t^T,
// Delta z = sum_t gamma^(last-t) phi(k_t), over the tokens of one segment.
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kThreads, 1)
summary_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const float* __restrict__ gamma, float* __restrict__ ws, int N, int H, int G, int L)
{
    using P = SummaryPlan<D, DV>;
    grid_launch_dependents();   // the scan may launch now; it waits for this grid's results
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    uint64_t* done = empty + P::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const float lam = DECAY ? logf(gamma[chain % H]) : 0.f;
    const uint64_t pol = policy_evict_last();  // the chunk kernel reads k, v again

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    // the ones-column tile of every stage: element (t, 0) = 1, the rest 0
    for (int s = 0; s < P::STAGES; ++s)
        for (int e = tid; e < C * 8; e += kThreads) {
            const int row = e / 8, chunk = e % 8;
            // logical chunk 0 of row `row` sits at physical chunk row % 8
            const uint32_t w = chunk == (row & 7) ? 0x3F80u : 0u;   // bf16 1.0 in the low half
            reinterpret_cast<uint4*>(sm + s * P::STAGE + P::KB + P::VB)[e] = make_uint4(w, 0u, 0u, 0u);
        }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    int loads_issued = 0, loads_waited = 0, commits = 0;
    auto issue = [&](int c) {
        const int s = c % P::STAGES;
        unsigned char* st = sm + s * P::STAGE;
        mbar_expect_tx(&full[s], P::LOAD_BYTES);
        for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_k, b * 64, t0 + c * C, chain, &full[s], pol);
        for (int b = 0; b < DV / 64; ++b)
            tma_load_3d(st + P::KB + b * TILE, &tm_v, b * 64, t0 + c * C, chain, &full[s], pol);
        loads_issued = c + 1;
    };
    if (tid == 0)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);

    bool bad = false;
    const int last = t1 - 1;
    for (int c = 0; c < nch; ++c) {
        const int s = c % P::STAGES;
        const uint32_t ph = (c / P::STAGES) & 1;
        unsigned char* kt = sm + s * P::STAGE;
        unsigned char* vt = kt + P::KB;
        if (!mbar_wait(&full[s], ph, kErrTmaLoad)) bad = true;
        else loads_waited = c + 1;
        // K~_t = gamma^(last - t) phi(k_t), zero past the end of the sequence
        const int tc0 = t0 + c * C;
        for (int e = tid; e < (D / 8) * C; e += kThreads) {
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            uint4* p = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
            const int t = tc0 + row;
            const float w = t <= last ? (DECAY ? __expf((float)(last - t) * lam) : 1.f) : 0.f;
            float f[8];
            unpack8(*p, f);
#pragma unroll
            for (int x = 0; x < 8; x += 2) {
                const float2 y = phi2_fast(f[x], f[x + 1]);
                f[x] = y.x; f[x + 1] = y.y;
            }
            *p = pack8(f, w);
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
        if (tid == 0) {
            // [Delta S | Delta z] += K~^T [V | 1]   (M = d, N = dv + 16)
            tc_fence_after();
            const uint32_t ka = smem_u32(kt), va = smem_u32(vt);
            const uint32_t id_s = idesc_bf16_f32(D, P::NS, 1, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_S, sdesc_sw128(ka + ks * 2048, TILE, 1024),
                         sdesc_sw128(va + ks * 2048, TILE, 1024), id_s, (c > 0 || ks > 0));
            mma_commit(&empty[s]);
            if (c == nch - 1) mma_commit(done);
            commits = c + 1;
        }
        // refill the stage chunk c-1 used: its MMA was issued a whole chunk ago.
        // The other threads go on to phi of the next chunk meanwhile.
        if (tid == 0 && c >= 1 && c - 1 + P::STAGES < nch) {
            const int sp = (c - 1) % P::STAGES;
            if (!mbar_wait(&empty[sp], ((c - 1) / P::STAGES) & 1, kErrMma)) bad = true;
            else issue(c - 1 + P::STAGES);
        }
    }
    if (!bad && !mbar_wait(done, 0, kErrMma)) bad = true;
    tc_fence_after();
    float* slot = ws + (size_t)unit * (D * DV + D);
    if (!bad) {
        const int f = acc_row<D>(quad, lane);
#pragma unroll
        for (int gg = 0; gg < DV / 64; ++gg) {
            const int col0 = wg * (DV / 4) + gg * 16;
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
            tmem_ld_wait();
            if (f >= 0) {
                float4* dst = reinterpret_cast<float4*>(slot + (size_t)f * DV + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        // Delta z: accumulator column dv, one row (feature) per lane
        if (wg == 0) {
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + DV), v);
            tmem_ld_wait();
            if (f >= 0) slot[D * DV + f] = v[0];
        }
    }
    if (bad && tid == 0) {
        // Leave no copy or MMA in flight before releasing TMEM and exiting.
        for (int cc = loads_waited; cc < loads_issued; ++cc)
            mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
        if (commits > 0)
            mbar_wait(&empty[(commits - 1) % P::STAGES], ((commits - 1) / P::STAGES) & 1, kErrMma);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
    // Launched early behind the previous call's kernels (one sequence after
    // another), this grid reads none of their results, but it completes only
    // after them, so the stream still finishes the calls in order.
    grid_dependency_wait();
}

// ---------------------------------------------------------------------------
// Kernel B: scan of segment summaries.  In place: slot s <- state at the start
// of segment s; writes the final state (S_N, z_N).
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(256)
scan_kernel(float* __restrict__ ws, const float* __restrict__ gamma, const float* __restrict__ S0,
            const float* __restrict__ z0, float* __restrict__ S_out, float* __restrict__ z_out, int N, int H,
            int G, int L)
{
    constexpr int SLOT = D * DV + D;
    grid_launch_dependents();   // the chunk kernel may set up and load q, k, v meanwhile
    grid_dependency_wait();     // the segment summaries are complete
    const int chain = blockIdx.x;
    const int e = blockIdx.y * 256 + threadIdx.x;
    if (e >= SLOT) return;
    const float lam = DECAY ? logf(gamma[chain % H]) : 0.f;
    const bool isz = e >= D * DV;
    float acc;
    if (!isz) acc = S0 ? S0[(size_t)chain * D * DV + e] : 0.f;
    else acc = z0 ? z0[(size_t)chain * D + (e - D * DV)] : 0.f;
    float* base = ws + (size_t)chain * G * SLOT + e;
    const float full_dec = DECAY ? expf((float)L * lam) : 1.f;
    constexpr int BATCH = 8;
    for (int s0 = 0; s0 < G; s0 += BATCH) {
        float delta[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) delta[i] = (s0 + i < G) ? base[(size_t)(s0 + i) * SLOT] : 0.f;
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int s = s0 + i;
            if (s < G) {
                base[(size_t)s * SLOT] = acc;
                const int len = min(L, N - s * L);
                const float dec = DECAY ? (len == L ? full_dec : expf((float)len * lam)) : 1.f;
                acc = fmaf(dec, acc, delta[i]);
            }
        }
    }
    if (!isz) S_out[(size_t)chain * D * DV + e] = acc;
    else z_out[(size_t)chain * D + (e - D * DV)] = acc;
}

// ---------------------------------------------------------------------------
// Kernel C: the chunk loop of one (chain, segment) from its start state.
//
// The state is kept transposed in TMEM (S^T: lane = value index, column =
// key feature), exactly the layout of the A operand of a tf32 MMA, so the
// start-state read of every chunk is an MMA straight out of TMEM and the
// state never passes through the CUDA cores.  The normaliser z is carried as
// row 0 of a small accumulator fed by a constant "ones row" tile; the
// denominators (row sums of P~ plus Q^.z) are formed on the CUDA cores.
//
// Decay uses a scaled frame: with r the frame's reference position, the
// stored state is T = gamma^-(c0 - r) S(c0-1) at chunk start c0, key rows are
// written as K^_t = gamma^-(t+1-r) phi(k_t) and query rows read as
// Q^_t = gamma^(t+1-r) phi(q_t).  The frame moves (T is rescaled once) only
// when |lambda| (t - r) would exceed kFrameLimit.
//
// Roles: warps 0..15 ("workers") run the epilogues and phi; lane 0 of warp 16
// ("issuer") issues TMA and every MMA.  Chunk c, from barrier B1:
//   issuer:  store o(c-1); MMA1 P = phi(Q)phi(K)^T; MMA3 O^T = S^T Q^^T
//            (tf32, A in TMEM); MMA4 S^T += V^T K^ and MMA4d z += 1^T K^;
//            prefetch; [wait P~] MMA2 O^T += V^T P~^T; release the staging tile
//   workers: [P ready] mask/decay -> P~ and its row sums, signal;  phi(c+1)
//            in place (overlaps the MMA batch);  [state carry done] frame
//            move, z of c+1, Q^/K^ of c+1 and Q^.z;  [outputs ready] 1/den,
//            o = O^T/den -> staging tile                              -> B1
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kThreads + 32, ChunkPlan<D, DV, DECAY>::TWO_PER_SM ? 2 : 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const float* __restrict__ gamma, const float* __restrict__ ws, int N, int H, int G, int L, float eps)
{
    using P = ChunkPlan<D, DV, DECAY>;
    constexpr int NCHK = (D / 8) * C / kThreads;  // 16-byte chunks of a Q (or K) tile per worker thread
    static_assert(NCHK >= 1 && (D / 8) * C % kThreads == 0, "tile split");
    grid_launch_dependents();   // a following call's summary pass may start as this grid drains
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* khat = sm + P::OFF_KH;
    unsigned char* q32 = sm + P::OFF_Q32;
    unsigned char* ptil = sm + P::OFF_P;
    unsigned char* ones = sm + P::OFF_ONES;
    unsigned char* otil = sm + P::OFF_O;
    float* rden = reinterpret_cast<float*>(sm + P::OFF_RDEN);
    float* dtab = reinterpret_cast<float*>(sm + P::OFF_DTAB);
    float* rsp = reinterpret_cast<float*>(sm + P::OFF_RSP);
    float* dint = reinterpret_cast<float*>(sm + P::OFF_DINT);
    float* zs = reinterpret_cast<float*>(sm + P::OFF_ZS);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* bar_p = full + P::STAGES;
    uint64_t* bar_s = bar_p + 1;
    uint64_t* bar_o = bar_p + 2;
    uint64_t* pt_full = bar_p + 3;
    uint64_t* o_free = bar_p + 4;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = warp >> 2;
    const bool worker = tid < kThreads;        // warps 0..15: epilogues and phi
    const bool issuer = tid == kThreads;       // lane 0 of warp 16: TMA and MMA issue
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const float lam = DECAY ? logf(gamma[chain % H]) : 0.f;
    const uint64_t pol_in = policy_evict_first();
    // One chunk's key weights reach gamma^-C; beyond e^80 they would overflow.
    if (DECAY && tid == 0 && (float)C * fabsf(lam) > 80.f) atomicCAS(&g_device_error, 0u, (unsigned int)kErrRange);

    if (tid == 0) {
        for (int s = 0; s < P::STAGES + 3; ++s) mbar_init(&full[s], 1);
        mbar_init(pt_full, kThreads / 32);
        mbar_init(o_free, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    if (tid < C) dtab[tid] = DECAY ? __expf((float)tid * lam) : 1.f;   // gamma^(i-j)
    if (tid < 8) {
        const uint32_t one2 = pack_bf16x2(1.f, 1.f);
        reinterpret_cast<uint4*>(ones)[tid] = make_uint4(one2, one2, one2, one2);   // row 0 only
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    // bookkeeping for the error path (meaningful in the issuer)
    int loads_issued = 0, commits = 0, commits_o = 0;
    int ref = 0;  // frame reference position (segment-local)
    auto chunk_len = [&](int c) { return min(C, t1 - (t0 + c * C)); };
    auto issue = [&](int c) {
        const int s = c % P::STAGES;
        unsigned char* st = sm + s * P::STAGE;
        const int y = t0 + c * C;
        loads_issued = c + 1;
        mbar_expect_tx(&full[s], P::STAGE);
        for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_q, b * 64, y, chain, &full[s], pol_in);
        for (int b = 0; b < D / 64; ++b)
            tma_load_3d(st + P::QB + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol_in);
        for (int b = 0; b < DV / 64; ++b)
            tma_load_3d(st + P::QB + P::KB + b * TILE, &tm_v, b * 64, y, chain, &full[s], pol_in);
    };
    // phi on load, part A: phi(q), phi(k) of chunk c into registers and, as
    // bf16, back in place (the score MMA operands; K zeroed past the end).
    float fq[NCHK][8], fk[NCHK][8];
    auto phi_a = [&](int c) {
        const int n = chunk_len(c);
        unsigned char* qt = sm + (c % P::STAGES) * P::STAGE;
        unsigned char* kt = qt + P::QB;
#pragma unroll
        for (int u = 0; u < NCHK; ++u) {
            const int e = tid + u * kThreads;
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            uint4* pq = reinterpret_cast<uint4*>(qt + b * TILE) + rem;
            uint4* pk = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
            unpack8(*pq, fq[u]);
            unpack8(*pk, fk[u]);
#pragma unroll
            for (int x = 0; x < 8; x += 2) {
                const float2 a = phi2_fast(fq[u][x], fq[u][x + 1]);
                const float2 b = phi2_fast(fk[u][x], fk[u][x + 1]);
                fq[u][x] = a.x; fq[u][x + 1] = a.y;
                fk[u][x] = b.x; fk[u][x + 1] = b.y;
            }
            *pq = pack8(fq[u], 1.f);
            *pk = pack8(fk[u], row < n ? 1.f : 0.f);
        }
    };
    // part B: the frame-weighted operands Q^ (fp32, tf32 MMA) and K^ (bf16),
    // and Q^ . z(c) for the denominators (8 consecutive threads share a row).
    auto phi_b = [&](int c) {
        const int n = chunk_len(c);
        const int c0 = c * C;
        const float* zc = zs + (c & 1) * D;
        float qz = 0.f;
#pragma unroll
        for (int u = 0; u < NCHK; ++u) {
            const int e = tid + u * kThreads;
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            const int f0 = b * 64 + (((rem % 8) ^ (row & 7)) * 8);   // first feature of this 16-byte chunk
            const float qw = DECAY ? __expf((float)(c0 + row + 1 - ref) * lam) : 1.f;
            unsigned char* qrow = q32 + (f0 / 32) * TILE;
            const int fb = (f0 % 32) * 4;
            *reinterpret_cast<float4*>(qrow + sw128_offset(row, fb)) =
                make_float4(qw * fq[u][0], qw * fq[u][1], qw * fq[u][2], qw * fq[u][3]);
            *reinterpret_cast<float4*>(qrow + sw128_offset(row, fb + 16)) =
                make_float4(qw * fq[u][4], qw * fq[u][5], qw * fq[u][6], qw * fq[u][7]);
            const float4 z0 = *reinterpret_cast<const float4*>(zc + f0);
            const float4 z1 = *reinterpret_cast<const float4*>(zc + f0 + 4);
            const float zz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
            for (int x = 0; x < 8; ++x) qz = fmaf(qw * fq[u][x], zz[x], qz);
            if (DECAY) {
                const float kw = row < n ? __expf(-(float)(c0 + row + 1 - ref) * lam) : 0.f;
                reinterpret_cast<uint4*>(khat + b * TILE)[rem] = pack8(fk[u], kw);
            }
        }
        qz += __shfl_xor_sync(0xffffffffu, qz, 1);
        qz += __shfl_xor_sync(0xffffffffu, qz, 2);
        qz += __shfl_xor_sync(0xffffffffu, qz, 4);
        if ((tid & 7) == 0) dint[(c & 1) * C + tid / 8] = qz;   // row tid/8 for every u
    };
    // Move the frame to position c0 (decay): S^T and z row times gamma^(c0 - ref).
    auto frame_move = [&](int c0) {
        const float m = __expf((float)(c0 - ref) * lam);
#pragma unroll
        for (int gg = 0; gg < D / 64; ++gg) {
            const int col0 = wg * (D / 4) + gg * 16;
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] *= m;
            tmem_st16(tmem_addr(tbase, quad, P::T_S + col0), v);
            tmem_ld16(tmem_addr(tbase, quad, P::T_Z + col0), v);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] *= m;
            tmem_st16(tmem_addr(tbase, quad, P::T_Z + col0), v);
        }
        tmem_st_wait();
    };
    // z at the start of chunk c (row 0 of the normaliser accumulator, lane 0
    // of quadrant 0) into zs[c & 1]; the caller synchronises the workers.
    auto z_to_smem = [&](int c) {
        if (quad == 0) {
#pragma unroll
            for (int gg = 0; gg < D / 64; ++gg) {
                const int col0 = wg * (D / 4) + gg * 16;
                float v[16];
                tmem_ld16(tmem_addr(tbase, 0, P::T_Z + col0), v);
                tmem_ld_wait();
                if (lane == 0) {
                    float4* dst = reinterpret_cast<float4*>(zs + (c & 1) * D + col0);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) dst[q4] = make_float4(v[4 * q4], v[4 * q4 + 1], v[4 * q4 + 2], v[4 * q4 + 3]);
                }
            }
        }
    };
    auto needs_move = [&](int c) {
        if (!DECAY) return false;
        return (float)(c * C + C - ref) * fabsf(lam) > kFrameLimit;
    };

    if (issuer)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);

    // Start state, transposed into TMEM: S^T[j][f] = S[f][j]; z as row 0 of
    // the normaliser accumulator (other rows zero).
    if (worker) {
        grid_dependency_wait();   // start states from the scan
        const float* slot = ws + (size_t)unit * (D * DV + D);
        const int j = acc_row<DV>(quad, lane);
#pragma unroll
        for (int gg = 0; gg < D / 64; ++gg) {
            const int col0 = wg * (D / 4) + gg * 16;
            float v[16];
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = j >= 0 ? slot[(size_t)(col0 + x) * DV + j] : 0.f;
            tmem_st16(tmem_addr(tbase, quad, P::T_S + col0), v);
#pragma unroll
            for (int x = 0; x < 16; ++x) v[x] = (quad == 0 && lane == 0) ? slot[D * DV + col0 + x] : 0.f;
            tmem_st16(tmem_addr(tbase, quad, P::T_Z + col0), v);
        }
        tmem_st_wait();
        if (tid < D) zs[tid] = slot[D * DV + tid];
        named_bar(5, kThreads);
    }
    bool bad = false;
    if (!mbar_wait(&full[0], 0, kErrTmaLoad)) bad = true;
    if (!bad && worker) {
        phi_a(0);
        phi_b(0);
    }
    fence_async_smem();
    tc_fence_before();
    if (__syncthreads_or(bad)) bad = true;

    for (int c = 0; c < nch && !bad; ++c) {
        const int s = c % P::STAGES;
        const uint32_t cp = c & 1;
        unsigned char* qt = sm + s * P::STAGE;
        unsigned char* kt = qt + P::QB;
        unsigned char* vt = kt + P::KB;
        unsigned char* kh = DECAY ? khat : kt;

        if (issuer) {
            tc_fence_after();
            if (c >= 1) {
                for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (c - 1) * C, chain);
                tma_store_commit();
            }
            const uint64_t dq = sdesc_sw128(smem_u32(qt), 16, 1024);      // K-major tiles
            const uint64_t dk = sdesc_sw128(smem_u32(kt), 16, 1024);
            const uint64_t dq32 = sdesc_sw128(smem_u32(q32), 16, 1024);
            const uint64_t dones = sdesc_sw128(smem_u32(ones), 16, 1024);
            const uint64_t dp = sdesc_sw128(smem_u32(ptil), 16, 1024);
            const uint64_t dv_mn = sdesc_sw128(smem_u32(vt), TILE, 1024);  // MN-major tiles
            const uint64_t dkh_mn = sdesc_sw128(smem_u32(kh), TILE, 1024);
            const uint32_t id1 = idesc_bf16_f32(64, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_P, dq + off, dk + off, id1, ks > 0);
            }
            mma_commit(bar_p);
            // start-state read, tf32 with S^T from TMEM (before MMA4 updates it)
            const uint32_t id3 = idesc_tf32_f32(DV, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 8; ++ks) {
                const uint64_t b = dq32 + (((ks / 4) * TILE + (ks % 4) * 32) >> 4);
                mma_tf32_ts(tbase + P::T_O, tbase + P::T_S + ks * 8, b, id3, ks > 0);
            }
            // state carry
            const uint32_t id4 = idesc_bf16_f32(DV, D, 1, 1);
            const uint32_t id4d = idesc_bf16_f32(64, D, 0, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t bk = dkh_mn + ((ks * 2048) >> 4);
                mma_bf16(tbase + P::T_S, dv_mn + ((ks * 2048) >> 4), bk, id4, 1u);
                mma_bf16(tbase + P::T_Z, dones + ((ks * 32) >> 4), bk, id4d, 1u);
            }
            mma_commit(bar_s);
            commits = c + 1;
            if (c >= 1 && c - 1 + P::STAGES < nch) issue(c - 1 + P::STAGES);
            // intra-chunk values once the workers have written P~
            if (!mbar_wait(pt_full, cp, kErrMma)) bad = true;
            tc_fence_after();
            const uint32_t id2 = idesc_bf16_f32(DV, 64, 1, 0);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_O, dv_mn + ((ks * 2048) >> 4), dp + ((ks * 32) >> 4), id2, 1u);
            mma_commit(bar_o);
            commits_o = c + 1;
            tma_store_wait_read();   // the staging tile may be rewritten
            mbar_arrive(o_free);
        }

        if (worker) {
            // scores -> P~: rows i (M=64 layout), columns split by warpgroup
            if (!mbar_wait(bar_p, cp, kErrMma)) bad = true;
            tc_fence_after();
            {
                const int i = acc_row<64>(quad, lane);
                float v[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_P + wg * 16), v);
                tmem_ld_wait();
                if (i >= 0) {
                    uint32_t pk[8];
                    float rs = 0.f;
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const int j0 = wg * 16 + 2 * h;
                        const float a = j0 <= i ? (DECAY ? v[2 * h] * dtab[i - j0] : v[2 * h]) : 0.f;
                        const float b = j0 + 1 <= i ? (DECAY ? v[2 * h + 1] * dtab[i - j0 - 1] : v[2 * h + 1]) : 0.f;
                        pk[h] = pack_bf16x2(a, b);
                        const float2 r = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[h]));
                        rs += r.x + r.y;   // the row sum of exactly the values the MMA uses
                    }
                    rsp[wg * C + i] = rs;
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(i, wg * 32)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(i, wg * 32 + 16)) =
                        make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pt_full);

            // phi of the next chunk, overlapping the MMA batch of this one
            const bool more = c + 1 < nch;
            const bool move = more && needs_move(c + 1);
            if (more) {
                if (!mbar_wait(&full[(c + 1) % P::STAGES], ((c + 1) / P::STAGES) & 1, kErrTmaLoad)) bad = true;
                else phi_a(c + 1);
            }
            // the state carry (and its reads of Q^ / K^) must be complete
            if (!mbar_wait(bar_s, cp, kErrMma)) bad = true;
            tc_fence_after();
            if (move) {
                frame_move((c + 1) * C);
                ref = (c + 1) * C;
            }
            if (more) {
                z_to_smem(c + 1);
                named_bar(5, kThreads);   // z(c+1) and every row sum of P~(c) are in smem
                phi_b(c + 1);
            } else {
                named_bar(5, kThreads);
            }

            // denominators: row 0 of the normaliser accumulator (lane 0, quadrant 0)
            if (!mbar_wait(bar_o, cp, kErrMma)) bad = true;
            tc_fence_after();
            if (quad == 0 && lane < 16) {
                const int i = wg * 16 + lane;
                const float den = rsp[i] + rsp[C + i] + rsp[2 * C + i] + rsp[3 * C + i] + dint[cp * C + i];
                rden[i] = __frcp_rn(den + eps);
            }
            named_bar(1 + wg, 128);   // this warpgroup's 16 denominators are in smem
            if (!mbar_wait(o_free, cp, kErrMma)) bad = true;
            // outputs o_i = O^T[:, i] / den_i -> staging tile (one value column per thread)
            {
                const int j = acc_row<DV>(quad, lane);
                float v[16], r[16];
                tmem_ld16(tmem_addr(tbase, quad, P::T_O + wg * 16), v);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 t = reinterpret_cast<const float4*>(rden + wg * 16)[q4];
                    r[4 * q4] = t.x; r[4 * q4 + 1] = t.y; r[4 * q4 + 2] = t.z; r[4 * q4 + 3] = t.w;
                }
                tmem_ld_wait();
                if (j >= 0) {
                    // element (i, j) of the swizzled staging tile: 16-byte chunk
                    // (j % 64) / 8 of row i, XOR (i % 8); i % 8 == x % 8 here
                    unsigned char* base = otil + (j / 64) * TILE + (j % 8) * 2;
                    const int cj = (j % 64) >> 3;
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int i = wg * 16 + x;
                        *reinterpret_cast<__nv_bfloat16*>(base + i * 128 + ((cj ^ (x & 7)) << 4)) =
                            __float2bfloat16_rn(v[x] * r[x]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }                         // B1
    }
    if (issuer) {
        if (!bad && nch > 0) {
            tc_fence_after();
            for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (nch - 1) * C, chain);
            tma_store_commit();
        }
        tma_store_wait_all();
        if (bad) {
            // Leave no copy or MMA in flight before releasing TMEM and exiting:
            // only the last STAGES loads can still be in flight.
            for (int cc = max(0, loads_issued - P::STAGES); cc < loads_issued; ++cc)
                mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
            if (commits > 0) {
                const uint32_t last = (commits - 1) & 1;
                mbar_wait(bar_p, last, kErrMma);
                mbar_wait(bar_s, last, kErrMma);
                if (commits_o > 0) mbar_wait(bar_o, (commits_o - 1) & 1, kErrMma);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
}

// ---------------------------------------------------------------------------
// host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

}  // namespace

// 3-D map over the first N rows of each chain of a bf16 [chains][ld][inner]
// tensor; box = 64 elements x 64 rows, 128-byte swizzle; rows past N read as
// zero and are not written.
bool make_map(CUtensorMap* m, const void* base, int inner, int N, int chains, int ld)
{
    auto fn = encode_fn();
    if (!fn || ld < N) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)chains};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)ld * inner * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <int D, int DV, bool DECAY>
cudaError_t launch_tc(const PrefillArgs& a, const TcSegments& sg)
{
    const int chains = a.B * a.H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, D, a.N, chains, a.ld) || !make_map(&mk, a.k, D, a.N, chains, a.ld) ||
        !make_map(&mv, a.v, DV, a.N, chains, a.ld) || !make_map(&mo, a.out, DV, a.N, chains, a.ld))
        return cudaErrorInvalidValue;
    float* ws = static_cast<float*>(a.workspace);
    const int units = chains * sg.G;

    auto ka = summary_kernel<D, DV, DECAY>;
    const int sa = SummaryPlan<D, DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, sa);
    if (e != cudaSuccess) return e;
    // all of L1 as shared memory, so that two CTAs fit on an SM where their plans allow
    e = cudaFuncSetAttribute(ka, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    // the scan and the chunk kernel (and, behind an earlier call of the same
    // batch, the summary pass) start with programmatic serialization: each
    // sets up while its predecessor finishes and waits only before reading
    // what the predecessor wrote (griddepcontrol.wait)
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(units);
    lc.blockDim = dim3(kThreads);
    lc.dynamicSmemBytes = sa;
    lc.stream = a.stream;
    lc.attrs = pdl;
    lc.numAttrs = a.pdl_first ? 1 : 0;
    e = cudaLaunchKernelEx(&lc, ka, mk, mv, a.gamma, ws, a.N, a.H, sg.G, sg.L);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(0, a.stream);

    constexpr int SLOT = D * DV + D;
    lc.gridDim = dim3(chains, (SLOT + 255) / 256);
    lc.blockDim = dim3(256);
    lc.dynamicSmemBytes = 0;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, scan_kernel<D, DV, DECAY>, ws, a.gamma, a.S0, a.z0, a.S_out, a.z_out, a.N, a.H,
                           sg.G, sg.L);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(1, a.stream);

    auto kc = chunk_kernel<D, DV, DECAY>;
    const int sc = ChunkPlan<D, DV, DECAY>::BYTES;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, sc);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    lc.gridDim = dim3(units);
    lc.blockDim = dim3(kThreads + 32);
    lc.dynamicSmemBytes = sc;
    e = cudaLaunchKernelEx(&lc, kc, mq, mk, mv, mo, a.gamma, (const float*)ws, a.N, a.H, sg.G, sg.L, a.eps);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(2, a.stream);
    return cudaSuccess;
}

}  // namespace

TcSegments tc_segments(int B, int H, int N, int d, int dv)
{
    TcSegments s;
    const long long chains = (long long)B * H;
    if (N <= 0 || chains <= 0) return s;
    // One CTA (two for d = dv = 64) per SM runs one segment at a time.  Prefer
    // whole waves of long segments: G segments per chain with chains * G close
    // to a multiple of the resident CTA count, and segments of at most kMaxSeg
    // tokens.
    constexpr long long kMaxSeg = 4096;
    const long long kSMs = (d == 64 && dv == 64) ? 2 * 148 : 148;
    long long G = 1, L = N;
    for (long long waves = 1;; ++waves) {
        G = waves * kSMs / chains;
        if (G < 1) G = 1;
        L = (N + G - 1) / G;
        L = ((L + C - 1) / C) * C;
        if (L <= kMaxSeg || L <= C) break;
    }
    if (L < 2 * C) L = 2 * C;
    s.L = (int)L;
    s.G = (int)((N + L - 1) / L);
    return s;
}

size_t tc_workspace_bytes(int B, int H, int N, int d, int dv)
{
    const TcSegments s = tc_segments(B, H, N, d, dv);
    return (size_t)B * H * s.G * ((size_t)d * dv + d) * sizeof(float);
}

cudaError_t launch_prefill_tc_kernelized(const PrefillArgs& a)
{
    const TcSegments sg = tc_segments(a.B, a.H, a.N, a.d, a.dv);
    const bool dec = a.mode == LA_DECAY;
#define LA_TC(D, DV)                                                               \
    if (a.d == D && a.dv == DV) return dec ? launch_tc<D, DV, true>(a, sg) : launch_tc<D, DV, false>(a, sg);
    LA_TC(64, 64)
    LA_TC(64, 128)
    LA_TC(128, 64)
    LA_TC(128, 128)
#undef LA_TC
    return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// No-allocation variant.  Some callers cannot call cudaMalloc on their launch
// path (an inference server that plans all device memory up front, a plugin
// host that hands out no workspace, code that must not trigger the implicit
// device synchronisation an allocation can cause).  For them the segment
// summaries live in this fixed array instead of a caller workspace.  Every
// GPU that loads the library holds it until the process exits.  All calls
// share it: calls whose work overlaps on the GPU (two streams, or two host
// threads) race on its contents and must be serialised by the caller.  The
// kernels overwrite every byte they later read, so nothing needs clearing.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// Device address of g_noalloc_scratch for the current device, looked up once
// per device with that device current.  In host code the symbol itself is
// only a host-side stand-in and must never be handed to a kernel.
void* noalloc_scratch_address(cudaError_t* err)
{
    static std::mutex mu;
    static void* addr[64] = {};
    int dev = -1;
    *err = cudaGetDevice(&dev);
    if (*err != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *err = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (*err != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

// Segment split that fits the fixed scratch: start from the usual split and
// lengthen segments until chains * segments summaries fit.  G == 0 means the
// problem is too large even with one segment per chain.
TcSegments tc_segments_noalloc(int B, int H, int N, int d, int dv)
{
    TcSegments s = tc_segments(B, H, N, d, dv);
    const size_t per_seg = (size_t)B * H * ((size_t)d * dv + d) * sizeof(float);
    if (per_seg == 0 || N == 0) return s;
    const size_t gmax = kNoAllocScratchBytes / per_seg;
    if (gmax == 0) {
        s.G = 0;
        return s;
    }
    if ((size_t)s.G > gmax) {
        long long L = ((long long)N + (long long)gmax - 1) / (long long)gmax;
        L = ((L + C - 1) / C) * C;
        s.L = (int)L;
        s.G = (int)((N + L - 1) / L);
    }
    return s;
}

cudaError_t launch_prefill_tc_kernelized_noalloc(const PrefillArgs& in)
{
    const TcSegments sg = tc_segments_noalloc(in.B, in.H, in.N, in.d, in.dv);
    if (sg.G == 0) return cudaErrorInvalidValue;
    cudaError_t e;
    void* scratch = noalloc_scratch_address(&e);
    if (!scratch) return e;
    PrefillArgs a = in;
    a.workspace = scratch;
    a.workspace_bytes = kNoAllocScratchBytes;
    const bool dec = a.mode == LA_DECAY;
#define LA_TC(D, DV)                                                               \
    if (a.d == D && a.dv == DV) return dec ? launch_tc<D, DV, true>(a, sg) : launch_tc<D, DV, false>(a, sg);
    LA_TC(64, 64)
    LA_TC(64, 128)
    LA_TC(128, 64)
    LA_TC(128, 128)
#undef LA_TC
    return cudaErrorInvalidValue;
}

unsigned int read_and_clear_device_error(cudaStream_t stream)
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
