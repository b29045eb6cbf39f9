// Tensor-core (tcgen05 + TMEM + TMA) prefill for the kernelized modes
// (LA_PLAIN, LA_DECAY) with bf16 inputs.
//
// Method ("What Is Linear Attention?" §4/§5.1; "Efficient attention
// variants" §5, §7.1 and §8 "chunkwise": parallel inside a chunk, state passed
// between chunks).  For a chunk of C = 64 tokens with start state (S, z),
// local positions i, j, lambda = log gamma_h and the chunk's middle m = 32:
//   Q~_i = gamma^(i-m) phi(q_i),   K~_j = gamma^(m-j) phi(k_j) [j < n]
//   P~   = [j <= i] (Q~ K~^T)_ij = [j <= i] gamma^(i-j) phi(q_i).phi(k_j)
//   o_i  = (P~ V + gamma^(i+1) phi(q_i)^T S)_i / (P~ 1 + gamma^(i+1) phi(q_i).z + eps)
//   S   <- gamma^C S + sum_j gamma^(C-1-j) phi(k_j) v_j^T,  z likewise
// (n valid tokens; the causal mask is multiplicative, "Transformers Are RNNs"
// notes).  The state is carried in a scaled frame T = S / kappa, kappa =
// gamma^(C-1-m), in which the carry reads T <- gamma^C T + K~^T V and the
// start-state read is Q~ (gamma^C T): the same operands Q~, K~ serve all three
// products, and no weight exceeds gamma^-32.
//
// Every contraction runs on the tensor cores, with the normaliser carried as
// a column of ones appended to V ([V | 1]) and to the state ([T | t_z]):
//   MMA1  P      = Q~ K~^T                  M=64, N=64,    K=d
//   MMA3  O      = Q~ [W | w_z],  W = gamma^C T (bf16 copy)   M=64, N=dv+16, K=d
//   MMA2  O     += P~ [V | 1]               M=64, N=dv+16, K=64
//   MMA4  [T|t_z] = [W|w_z] + K~^T [V | 1]   M=d,  N=dv+16, K=64  (fp32 in TMEM)
// so column dv of O is the denominator, and each output row is divided and
// stored as whole 16-byte pieces.
//
// Parallelism across the sequence ("Transformers Are RNNs" notes: the state
// is a prefix sum, so it can be scanned): each (chain, segment) of L tokens
// is one CTA.  Kernel A reduces every segment to its summary
// (Delta S, Delta z); kernel B scans summaries into segment start states and
// the final state; kernel C runs the chunk loop of every segment from its
// true start state.
//
// Supported decay range on this path: 32 |log gamma| <= 73.7 (gamma >= 0.1);
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

// ---------------------------------------------------------------------------
// Shared-memory plan of the chunk kernel (all tiles 1024-byte aligned).
template <int D, int DV, bool DECAY>
struct ChunkPlan {
    // d = dv = 64: two CTAs share an SM, so one CTA's waits hide behind the other's work
    static constexpr bool TWO_PER_SM = D == 64 && DV == 64;
    // worker warps: a TMEM group of NT (every lane quadrant) and a phi group of
    // NW - NT; with the issuer warp a CTA has 16 (two per SM: 8) warps, four
    // (two) per SM sub-partition, which leaves 128 registers a thread
    static constexpr int NW = TWO_PER_SM ? 7 : 15;
    static constexpr int NT = TWO_PER_SM ? 4 : 8;
    static constexpr int THREADS = (NW + 1) * 32;          // + the issuer warp
    static constexpr int STAGES = 2;
    static constexpr int NO = DV + 16;                     // accumulator columns of O and T
    static constexpr int NBLK = DV / 64 + 1;               // 64-column blocks of [V | 1]
    // stage: Q~ tiles | K~ tiles | V tiles | ones tile (column 0 = 1): [V | 1] is one
    // MN-major B operand whose 64-column blocks are a tile apart
    static constexpr int QB = C * D * 2, KB = C * D * 2, VB = C * DV * 2;
    static constexpr int LOAD_BYTES = QB + KB + VB;
    static constexpr int STAGE = QB + KB + VB + TILE;
    static constexpr int OFF_W = STAGES * STAGE;           // [W | w_z] bf16, NBLK blocks of D x 64
    static constexpr int WBLK = D * 128;
    static constexpr int OFF_P = OFF_W + NBLK * WBLK;      // P~ bf16 [C][C]
    static constexpr int OFF_O = OFF_P + TILE;             // output staging bf16 [C][DV]
    static constexpr int OFF_WT = OFF_O + C * DV * 2;      // [4][C] fp32 decay weights of Q~, K~ and their log2
    static constexpr int OFF_BAR = OFF_WT + 4 * C * 4;
    // full[S] empty[S] phi[S] w_ready t_done p_full ptil o_full o_read os_full os_empty drain
    static constexpr int NBAR = 3 * STAGES + 9;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;     // + alignment slack
    static_assert(BYTES <= 232448, "shared memory plan exceeds the per-block limit");
    static_assert(!TWO_PER_SM || 2 * (BYTES + 1024) <= 233472, "two CTAs per SM");
    // TMEM columns: scores, output (+ denominator), state (+ normaliser)
    static constexpr uint32_t T_P = 0, T_O = 64, T_T = 64 + NO;
    static constexpr uint32_t T_COLS = (T_T + NO <= 256) ? 256 : 512;
};

template <int D, int DV>
struct SummaryPlan {
    static constexpr int STAGES = 4;
    static constexpr int KB = C * D * 2, VB = C * DV * 2;
    // stage: K tiles, V tiles, then a constant tile whose column 0 is ones:
    // B = [V | 1] makes column dv of K~^T B the normaliser sum Delta z
    static constexpr int LOAD_BYTES = KB + VB;
    static constexpr int STAGE = KB + VB + TILE;
    static constexpr int OFF_BAR = STAGES * STAGE;                // full[S], empty[S], phi[S], done
    static constexpr int OFF_TMEM = OFF_BAR + (3 * STAGES + 1) * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static constexpr int NS = DV + 16;                            // accumulator columns
    static constexpr uint32_t T_S = 0, T_COLS = 256;
};


// ---------------------------------------------------------------------------
// Units of a segment map: one (chain, segment) each, with its token range.
struct Unit {
    int chain, t0, t1;
    bool clip;   // a sequence of a padded batch: rows past t1 may hold padding
};

__device__ __forceinline__ Unit unit_of(const SegMap& m, int unit)
{
    Unit u;
    if (m.B == 0) {
        const int seg = unit % m.G;
        u.chain = unit / m.G;
        u.t0 = seg * m.L;
        u.t1 = min(m.N, u.t0 + m.L);
        u.clip = false;
        return u;
    }
    int base = 0, b = 0;
    for (; b < m.B; ++b) {
        const int n = m.H * ((m.lens[b] + m.L - 1) / m.L);
        if (unit < base + n) break;
        base += n;
    }
    const int g = (m.lens[b] + m.L - 1) / m.L;
    const int r = unit - base;
    u.chain = b * m.H + r / g;
    u.t0 = (r % g) * m.L;
    u.t1 = min(m.lens[b], u.t0 + m.L);
    u.clip = true;
    return u;
}

__device__ __forceinline__ int chunk_len_of(int t0, int t1, int c) { return min(C, t1 - (t0 + c * C)); }

// First slot, segment count and token count of chain c.
__device__ __forceinline__ void chain_of(const SegMap& m, int c, int& slot0, int& g, int& n)
{
    if (m.B == 0) {
        slot0 = c * m.G;
        g = m.G;
        n = m.N;
        return;
    }
    const int b = c / m.H, h = c % m.H;
    int base = 0;
    for (int i = 0; i < b; ++i) base += m.H * ((m.lens[i] + m.L - 1) / m.L);
    n = m.lens[b];
    g = (n + m.L - 1) / m.L;
    slot0 = base + h * g;
}

// Zero the value rows n..C-1 of a chunk's V tiles (a padded batch's padding may
// hold anything, and a zero weight times a non-finite value is not zero).
template <int DV>
__device__ __forceinline__ void zero_tail_rows(unsigned char* vt, int n, int tid, int nthreads)
{
    for (int e = tid; e < (DV / 8) * C; e += nthreads) {
        const int rem = e % (8 * C), row = rem / 8;
        if (row >= n) reinterpret_cast<uint4*>(vt)[e] = make_uint4(0u, 0u, 0u, 0u);
    }
}

// ---------------------------------------------------------------------------
// Kernel A: segment summaries  Delta S = sum_t gamma^(last-t) phi(k_t) v_t^T,
// Delta z = sum_t gamma^(last-t) phi(k_t), over the tokens of one segment.
//
// Roles: warps 0..15 apply phi (and the decay weight) to each stage's K in
// place and signal its per-stage barrier; lane 0 of warp 16 issues the TMA
// loads and the MMAs.  The phi warps run as far ahead as the loads allow, so
// their exponentials overlap the copies and the contraction.
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kThreads + 32, 1)
summary_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const float* __restrict__ gamma, float* __restrict__ ws, const __grid_constant__ SegMap m)
{
    using P = SummaryPlan<D, DV>;
    grid_launch_dependents();   // the scan may launch now; it waits for this grid's results
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    uint64_t* phi_rdy = empty + P::STAGES;   // phi warps: K~ of the stage's chunk in place
    uint64_t* done = phi_rdy + P::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, wg = (warp >> 2) & 3;
    const bool issuer = tid == kThreads;
    const int unit = blockIdx.x;
    const Unit un = unit_of(m, unit);
    const int chain = un.chain, t0 = un.t0, t1 = un.t1;
    const int nch = (t1 - t0 + C - 1) / C;
    const float lam = DECAY ? logf(gamma[chain % m.H]) : 0.f;
    const uint64_t pol = policy_evict_last();  // the chunk kernel reads k, v again

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&phi_rdy[s], kThreads / 32);
        }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    // the ones-column tile of every stage: element (t, 0) = 1, the rest 0
    for (int s = 0; s < P::STAGES; ++s)
        for (int e = tid; e < C * 8; e += kThreads + 32) {
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

    bool bad = false;
    if (issuer) {
        int loads = 0, commits = 0;
        auto issue = [&](int c) {
            const int s = c % P::STAGES;
            unsigned char* st = sm + s * P::STAGE;
            mbar_expect_tx(&full[s], P::LOAD_BYTES);
            for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_k, b * 64, t0 + c * C, chain, &full[s], pol);
            for (int b = 0; b < DV / 64; ++b)
                tma_load_3d(st + P::KB + b * TILE, &tm_v, b * 64, t0 + c * C, chain, &full[s], pol);
            loads = c + 1;
        };
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
        const uint32_t id_s = idesc_bf16_f32(D, P::NS, 1, 1);
        for (int c = 0; c < nch; ++c) {
            const int s = c % P::STAGES;
            if (!mbar_wait(&phi_rdy[s], (c / P::STAGES) & 1, kErrMma)) { bad = true; break; }
            tc_fence_after();
            // [Delta S | Delta z] += K~^T [V | 1]   (M = d, N = dv + 16)
            const uint32_t ka = smem_u32(sm + s * P::STAGE), va = ka + P::KB;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_S, sdesc_sw128(ka + ks * 2048, TILE, 1024),
                         sdesc_sw128(va + ks * 2048, TILE, 1024), id_s, (c > 0 || ks > 0));
            mma_commit(&empty[s]);
            if (c == nch - 1) mma_commit(done);
            commits = c + 1;
            // refill the stage chunk c-1 used: its MMA was issued a chunk ago
            if (c >= 1 && c - 1 + P::STAGES < nch) {
                if (!mbar_wait(&empty[(c - 1) % P::STAGES], ((c - 1) / P::STAGES) & 1, kErrMma)) { bad = true; break; }
                issue(c - 1 + P::STAGES);
            }
        }
        if (bad) {
            // leave no copy or MMA in flight before TMEM is released
            for (int cc = max(0, loads - P::STAGES); cc < loads; ++cc)
                mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
            if (commits > 0)
                mbar_wait(&empty[(commits - 1) % P::STAGES], ((commits - 1) / P::STAGES) & 1, kErrMma);
        }
    } else if (warp < kThreads / 32) {
        const int last = t1 - 1;
        for (int c = 0; c < nch; ++c) {
            const int s = c % P::STAGES;
            unsigned char* kt = sm + s * P::STAGE;
            unsigned char* vt = kt + P::KB;
            if (!mbar_wait(&full[s], (c / P::STAGES) & 1, kErrTmaLoad)) { bad = true; break; }
            if (un.clip && t1 - (t0 + c * C) < C) zero_tail_rows<DV>(vt, t1 - (t0 + c * C), tid, kThreads);
            // K~_t = gamma^(last - t) phi(k_t), zero past the end of the sequence:
            // w phi(x) = w max(x, 0) + 2^((x - max(x, 0)) log2 e + log2 w), the weight
            // riding in the exponent
            constexpr float kLog2e = 1.4426950408889634f;
            const int tc0 = t0 + c * C;
            for (int e = tid; e < (D / 8) * C; e += kThreads) {
                const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
                uint4* p = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
                const int t = tc0 + row;
                const float lw = DECAY ? (float)(last - t) * lam * kLog2e : 0.f;
                const float w = DECAY ? ex2_approx(lw) : 1.f;
                float f[8];
                unpack8(*p, f);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    const float mx = fmaxf(f[x], 0.f);
                    f[x] = fmaf(mx, w, ex2_approx(fmaf(f[x] - mx, kLog2e, lw)));
                }
                // rows past the end are stored as zeros: a padded batch's padding
                // may hold anything, and a zero weight times inf is not zero
                *p = t <= last ? pack8(f, 1.f) : make_uint4(0u, 0u, 0u, 0u);
            }
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&phi_rdy[s]);
        }
        if (!bad && !mbar_wait(done, 0, kErrMma)) bad = true;
    }
    // every thread agrees whether the summary is complete before it is read out
    const bool any_bad = __syncthreads_or(bad);
    tc_fence_after();
    float* slot = ws + (size_t)unit * (D * DV + D);
    if (!any_bad && warp < kThreads / 32) {
        const int f = acc_row<D>(quad, lane);
#pragma unroll
        for (int gg = 0; gg < DV / 64; ++gg) {
            const int col0 = wg * (DV / 4) + gg * 16;
            float v[16];
            tmem_ld16(tmem_addr(tbase, quad, P::T_S + col0), v);
            tmem_ld_wait();
            tmem_regs_after_wait(v);
            if (f >= 0) {
                float4* dst = reinterpret_cast<float4*>(slot + (size_t)f * DV + col0);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        // Delta z: accumulator column dv, one row (feature) per lane
        if (wg == 0) {
            float z = tmem_ld1(tmem_addr(tbase, quad, P::T_S + DV));
            tmem_ld_wait();
            tmem_regs_after_wait(z);
            if (f >= 0) slot[D * DV + f] = z;
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

// ---------------------------------------------------------------------------
// Kernel B: scan of segment summaries.  In place: slot s <- state at the start
// of segment s; writes the final state (S_N, z_N).  Every element is a short
// serial sum over its chain's segments.  Grid (chains, kScanSplit) of
// kScanThreads threads, each 16-byte column with eight segments' loads in
// flight: the scan holds few SMs, so the chunk kernel (launched behind it with
// programmatic serialization) becomes resident on the others and loads and
// applies phi to its first chunks while the scan runs.
constexpr int kScanThreads = 1024, kScanSplit = 4;

template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kScanThreads, 1)
scan_kernel(float* __restrict__ ws, const float* __restrict__ gamma, const float* __restrict__ S0,
            const float* __restrict__ z0, float* __restrict__ S_out, float* __restrict__ z_out,
            const __grid_constant__ SegMap m)
{
    constexpr int SLOT4 = (D * DV + D) / 4, S4 = D * DV / 4, BATCH = 8;
    grid_launch_dependents();   // the chunk kernel may set up and load q, k, v meanwhile
    grid_dependency_wait();     // the segment summaries are complete
    const int chain = blockIdx.x;
    int slot0, G, N;
    chain_of(m, chain, slot0, G, N);
    const int L = m.L;
    const float lam = DECAY ? logf(gamma[chain % m.H]) : 0.f;
    const float full_dec = DECAY ? expf((float)L * lam) : 1.f;
    float4* base = reinterpret_cast<float4*>(ws + (size_t)slot0 * (D * DV + D));
    const int per = (SLOT4 + gridDim.y - 1) / gridDim.y;   // columns of this CTA
    const int lo = blockIdx.y * per, hi = min(SLOT4, lo + per);
    for (int e = lo + (int)threadIdx.x; e < hi; e += kScanThreads) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < S4) { if (S0) acc = reinterpret_cast<const float4*>(S0 + (size_t)chain * D * DV)[e]; }
        else if (z0) acc = reinterpret_cast<const float4*>(z0 + (size_t)chain * D)[e - S4];
        for (int s0 = 0; s0 < G; s0 += BATCH) {
            float4 delta[BATCH];
#pragma unroll
            for (int i = 0; i < BATCH; ++i)
                delta[i] = (s0 + i < G) ? base[(size_t)(s0 + i) * SLOT4 + e] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int i = 0; i < BATCH; ++i) {
                const int sg = s0 + i;
                if (sg < G) {
                    base[(size_t)sg * SLOT4 + e] = acc;
                    const int len = min(L, N - sg * L);
                    const float dec = DECAY ? (len == L ? full_dec : expf((float)len * lam)) : 1.f;
                    acc.x = fmaf(dec, acc.x, delta[i].x);
                    acc.y = fmaf(dec, acc.y, delta[i].y);
                    acc.z = fmaf(dec, acc.z, delta[i].z);
                    acc.w = fmaf(dec, acc.w, delta[i].w);
                }
            }
        }
        if (e < S4) reinterpret_cast<float4*>(S_out + (size_t)chain * D * DV)[e] = acc;
        else reinterpret_cast<float4*>(z_out + (size_t)chain * D)[e - S4] = acc;
    }
}

// ---------------------------------------------------------------------------
// Kernel C: the chunk loop of one (chain, segment) from its start state.
//
// Roles: worker warps 0..NW-1 do the CUDA-core steps in two groups that run
// side by side; lane 0 of warp NW (the issuer) issues every TMA copy and every
// MMA.  Per chunk c:
//   TMEM group (warps 0..NT-1, every lane quadrant)
//            [t_done(c-1)] W = gamma^C T -> TMEM (decay) and bf16 -> smem;
//            [p_full(c)]   P~ = causal mask of P -> bf16;
//            [o_full(c)]   o = O / (O[:, dv] + eps) -> staging
//   phi group (warps NT..NW-1)
//            [full(c)]     phi, weights of chunk c in place (runs a chunk ahead)
//   issuer   [phi(c)] MMA1;  [w_ready(c), o_read(c-1)] MMA3, MMA4;
//            TMA store of chunk c-1;  [ptil(c)] MMA2;  loads of chunk c+2
// The state chain of a CTA is t_done(c-1) -> W copy -> MMA3, MMA4 -> t_done(c).
// phi is bound by the exponential unit and the TMEM steps by load latency, so
// the two groups fill each other's gaps.
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(ChunkPlan<D, DV, DECAY>::THREADS, ChunkPlan<D, DV, DECAY>::TWO_PER_SM ? 2 : 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const float* __restrict__ gamma, const float* __restrict__ ws, const __grid_constant__ SegMap m,
             float eps, __nv_bfloat16* __restrict__ out, int ld)
{
    using P = ChunkPlan<D, DV, DECAY>;
    constexpr int NW = P::NW;
    constexpr int NWT = NW * 32;                      // worker threads
    constexpr int NT = P::NT;                         // TMEM group: warps 0 .. NT-1
    constexpr int NTQ = NT / 4;                       // TMEM group warps per lane quadrant
    constexpr int NPT = (NW - NT) * 32;               // phi group threads (warps NT .. NW-1)
    grid_launch_dependents();   // a following call's summary pass may start as this grid drains
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* wcp = sm + P::OFF_W;
    unsigned char* ptil = sm + P::OFF_P;
    unsigned char* otil = sm + P::OFF_O;
    float* wq = reinterpret_cast<float*>(sm + P::OFF_WT);
    float* wk = wq + C;
    float* lwq = wq + 2 * C;
    float* lwk = wq + 3 * C;
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    // phi group: Q~, K~ of the stage's chunk in place.  One barrier per stage: the
    // phi group's warps run independently, and a warp that finished chunk c may
    // arrive for chunk c + 1 before the others arrived for chunk c.
    uint64_t* phi_rdy = empty + P::STAGES;
    uint64_t* w_rdy = phi_rdy + P::STAGES;   // TMEM group: W copy written (and T rescaled)
    uint64_t* t_done = w_rdy + 1;            // MMA3 + MMA4 complete
    uint64_t* p_full = w_rdy + 2;            // MMA1 complete
    uint64_t* ptil_rdy = w_rdy + 3;          // TMEM group: P~ written
    uint64_t* o_full = w_rdy + 4;            // MMA2 complete
    uint64_t* o_read = w_rdy + 5;            // TMEM group: O read out
    uint64_t* os_full = w_rdy + 6;           // TMEM group: output staging written
    uint64_t* os_empty = w_rdy + 7;          // issuer: staging read by its store
    uint64_t* drain = w_rdy + 8;             // issuer: every MMA it issued is complete
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool worker = warp < NW;
    const bool issuer = tid == NWT;
    const int quad = warp & 3;                        // TMEM lane quadrant
    const int unit = blockIdx.x;
    const Unit un = unit_of(m, unit);
    const int chain = un.chain, t0 = un.t0, t1 = un.t1;
    const int nch = (t1 - t0 + C - 1) / C;
    // a padded batch's last chunk of a sequence: its rows past the end hold
    // padding, so V's are zeroed and the output rows are stored one by one
    const bool clip_tail = un.clip && chunk_len_of(t0, t1, nch - 1) < C;
    const float lam = DECAY ? logf(gamma[chain % m.H]) : 0.f;
    const uint64_t pol_in = policy_evict_first();
    // the scaled frame keeps every weight within gamma^-32
    if (DECAY && tid == 0 && 32.f * fabsf(lam) > 73.7f) atomicCAS(&g_device_error, 0u, (unsigned int)kErrRange);

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        for (int s = 0; s < P::STAGES; ++s) mbar_init(&phi_rdy[s], NW - NT);
        mbar_init(w_rdy, NT);
        mbar_init(t_done, 1);
        mbar_init(p_full, 1);
        mbar_init(ptil_rdy, NT);
        mbar_init(o_full, 1);
        mbar_init(o_read, NT);
        mbar_init(os_full, NT);
        mbar_init(os_empty, 1);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    if (tid < C) {
        constexpr float kLog2e = 1.4426950408889634f;
        wq[tid] = DECAY ? __expf((float)(tid - C / 2) * lam) : 1.f;
        wk[tid] = DECAY ? __expf((float)(C / 2 - tid) * lam) : 1.f;
        lwq[tid] = DECAY ? (float)(tid - C / 2) * lam * kLog2e : 0.f;   // log2 of the weights
        lwk[tid] = DECAY ? (float)(C / 2 - tid) * lam * kLog2e : 0.f;
    }
    // the ones tile of every stage: element (t, 0) = 1, the rest 0
    for (int s = 0; s < P::STAGES; ++s)
        for (int e = tid; e < C * 8; e += P::THREADS) {
            const int row = e / 8, chunk = e % 8;
            const uint32_t one = chunk == (row & 7) ? 0x3F80u : 0u;   // bf16 1.0 in logical column 0
            reinterpret_cast<uint4*>(sm + s * P::STAGE + P::QB + P::KB + P::VB)[e] = make_uint4(one, 0u, 0u, 0u);
        }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    // gamma^C as two factors gamma^(C/2): gamma^C itself is below the fp32
    // range for gamma < 0.25, while gamma^C T is not
    const float gH = DECAY ? __expf((float)(C / 2) * lam) : 1.f;
    const bool one_factor = (float)C * fabsf(lam) < 80.f;   // gamma^C itself is a normal fp32
    const float gC = gH * gH;
    const float rkappa = DECAY ? __expf(-(float)(C - 1 - C / 2) * lam) : 1.f;   // 1 / kappa

    auto chunk_len = [&](int c) { return min(C, t1 - (t0 + c * C)); };
    bool bad = false;

    if (issuer) {
        // ---------------- issuer: TMA and MMA ----------------
        int loads = 0;
        auto issue = [&](int c) {
            const int s = c % P::STAGES;
            unsigned char* st = sm + s * P::STAGE;
            const int y = t0 + c * C;
            mbar_expect_tx(&full[s], P::LOAD_BYTES);
            for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_q, b * 64, y, chain, &full[s], pol_in);
            for (int b = 0; b < D / 64; ++b)
                tma_load_3d(st + P::QB + b * TILE, &tm_k, b * 64, y, chain, &full[s], pol_in);
            for (int b = 0; b < DV / 64; ++b)
                tma_load_3d(st + P::QB + P::KB + b * TILE, &tm_v, b * 64, y, chain, &full[s], pol_in);
            loads = c + 1;
        };
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);
        const uint32_t id1 = idesc_bf16_f32(64, 64, 0, 0);
        const uint32_t ido = idesc_bf16_f32(64, P::NO, 0, 1);
        const uint32_t idt = idesc_bf16_f32(D, P::NO, 1, 1);
        const uint64_t dw = sdesc_sw128(smem_u32(wcp), P::WBLK, 1024);
        const uint64_t dp = sdesc_sw128(smem_u32(ptil), 16, 1024);
        for (int c = 0; c < nch; ++c) {
            const int s = c % P::STAGES;
            const uint32_t cp = c & 1;
            unsigned char* st = sm + s * P::STAGE;
            const uint64_t dq = sdesc_sw128(smem_u32(st), 16, 1024);                 // Q~, K-major
            const uint64_t dk = sdesc_sw128(smem_u32(st + P::QB), 16, 1024);         // K~, K-major
            const uint64_t dkm = sdesc_sw128(smem_u32(st + P::QB), TILE, 1024);      // K~^T, MN-major
            const uint64_t dvb = sdesc_sw128(smem_u32(st + P::QB + P::KB), TILE, 1024);   // [V | 1]
            // MMA1: P = Q~ K~^T (P of the previous chunk was read before its P~ was signalled)
            if (!mbar_wait(&phi_rdy[s], (c / P::STAGES) & 1, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_P, dq + off, dk + off, id1, ks > 0);
            }
            mma_commit(p_full);
            // MMA3: O = Q~ [W | w_z];  MMA4: T = [W | w_z] (already in TMEM) + K~^T [V | 1]
            if (!mbar_wait(w_rdy, cp, kErrMma)) { bad = true; break; }
            if (c >= 1 && !mbar_wait(o_read, (c - 1) & 1, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = ((ks / 4) * TILE + (ks % 4) * 32) >> 4;
                mma_bf16(tbase + P::T_O, dq + off, dw + ((ks * 2048) >> 4), ido, ks > 0);
            }
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_T, dkm + ((ks * 2048) >> 4), dvb + ((ks * 2048) >> 4), idt, 1u);
            mma_commit(t_done);
            // the output of the previous chunk: its staging was written before W of
            // this chunk (the TMEM group's order), so the wait returns at once
            if (c >= 1) {
                if (!mbar_wait(os_full, (c - 1) & 1, kErrMma)) { bad = true; break; }
                fence_async_smem();
                for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (c - 1) * C, chain);
                tma_store_commit();
            }
            // MMA2: O += P~ [V | 1]
            if (!mbar_wait(ptil_rdy, cp, kErrMma)) { bad = true; break; }
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_O, dp + ((ks * 32) >> 4), dvb + ((ks * 2048) >> 4), ido, 1u);
            mma_commit(o_full);
            mma_commit(&empty[s]);
            // the staging is free once the store has read it (long done by now);
            // then the loads of chunk c + STAGES
            if (c >= 1) {
                tma_store_wait_read();
                mbar_arrive(os_empty);
            }
            if (c + P::STAGES < nch) {
                if (!mbar_wait(&empty[s], (c / P::STAGES) & 1, kErrMma)) { bad = true; break; }
                issue(c + P::STAGES);
            }
        }
        if (!bad && nch > 0 && mbar_wait(os_full, (nch - 1) & 1, kErrMma) && !clip_tail) {
            for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + (nch - 1) * C, chain);
            tma_store_commit();
        }
        tma_store_wait_all();
        // leave no copy or MMA in flight before TMEM is released
        for (int cc = max(0, loads - P::STAGES); cc < loads; ++cc)
            mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
        mma_commit(drain);
        mbar_wait(drain, 0, kErrMma);
    } else if (warp >= NT && warp < NW) {
        // ---------------- phi group: Q~, K~ of every chunk in place ----------------
        // w phi(x) = w max(x, 0) + 2^(min(x, 0) log2 e + log2 w): the operand weight rides in
        // the exponent (w = 0, for key rows past the sequence's end, gives exactly 0)
        const int ptid = tid - NT * 32;
        for (int c = 0; c < nch && !bad; ++c) {
            if (!mbar_wait(&full[c % P::STAGES], (c / P::STAGES) & 1, kErrTmaLoad)) { bad = true; break; }
            const int n = chunk_len(c);
            unsigned char* qt = sm + (c % P::STAGES) * P::STAGE;
            unsigned char* kt = qt + P::QB;
            constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll 1
            for (int e = ptid; e < (D / 8) * C; e += NPT) {
                const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
                uint4* pq = reinterpret_cast<uint4*>(qt + b * TILE) + rem;
                uint4* pk = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
                const bool kv = row < n;
                const float aq = DECAY ? wq[row] : 1.f, lq = DECAY ? lwq[row] : 0.f;
                const float ak = DECAY ? wk[row] : 1.f, lk = DECAY ? lwk[row] : 0.f;
                float fq[8], fk[8];
                unpack8(*pq, fq);
                unpack8(*pk, fk);
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    // min(x, 0) = x - max(x, 0) exactly: an add instead of a second min
                    const float mq = fmaxf(fq[x], 0.f), mk = fmaxf(fk[x], 0.f);
                    fq[x] = fmaf(mq, aq, ex2_approx(fmaf(fq[x] - mq, kLog2e, lq)));
                    fk[x] = fmaf(mk, ak, ex2_approx(fmaf(fk[x] - mk, kLog2e, lk)));
                }
                *pq = pack8(fq, 1.f);
                // key rows past the end are stored as zeros: a padded batch's padding
                // may hold anything, and a zero weight times inf is not zero
                *pk = kv ? pack8(fk, 1.f) : make_uint4(0u, 0u, 0u, 0u);
            }
            if (clip_tail && c == nch - 1) zero_tail_rows<DV>(kt + P::KB, n, ptid, NPT);
            fence_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&phi_rdy[c % P::STAGES]);
        }
    } else if (worker) {
        // ---------------- TMEM group: state copy, P~, output ----------------
        // NTQ warps per TMEM lane quadrant; warp `sub` of a quadrant takes the
        // 16-column groups sub, sub + NTQ, ...  Each batch of TMEM loads waits once.
        const int sub = warp >> 2;
        constexpr int KB = 1;       // TMEM loads per wait
        const int fr = acc_row<D>(quad, lane);      // state row of this thread (M = D accumulator)
        const int ir = acc_row<64>(quad, lane);     // score / output row (M = 64 accumulators)
        // W = gamma^C T of one 16-column group: into TMEM (the carry adds to it) and
        // as the bf16 B operand
        auto put_w = [&](int g, float (&v)[16], bool to_tmem) {
            if (DECAY) {
#pragma unroll
                for (int x = 0; x < 16; ++x) v[x] = one_factor ? v[x] * gC : (v[x] * gH) * gH;
            }
            if (to_tmem) tmem_st16(tmem_addr(tbase, quad, P::T_T + g * 16), v);
            if (fr >= 0) {
                unsigned char* blk = wcp + (g / 4) * P::WBLK;
                const int byte0 = (g % 4) * 32;
                *reinterpret_cast<uint4*>(blk + sw128_offset(fr, byte0)) =
                    make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7]));
                *reinterpret_cast<uint4*>(blk + sw128_offset(fr, byte0 + 16)) =
                    make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]), pack_bf16x2(v[12], v[13]),
                               pack_bf16x2(v[14], v[15]));
            }
        };
        auto w_ready = [&]() {
            tmem_st_wait();
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(w_rdy);
        };
        // chunk 0: T0 = S / kappa, the segment's start state from the scan (normaliser
        // as column dv), goes to TMEM and to W straight from the registers
        {
            grid_dependency_wait();
            const float* slot = ws + (size_t)unit * (D * DV + D);
#pragma unroll 1
            for (int g = sub; g < P::NO / 16; g += NTQ) {
                float v[16];
                if (g < DV / 16) {
                    const float4* src = reinterpret_cast<const float4*>(slot + (size_t)(fr >= 0 ? fr : 0) * DV + g * 16);
#pragma unroll
                    for (int x = 0; x < 4; ++x) {
                        const float4 t = fr >= 0 ? src[x] : make_float4(0.f, 0.f, 0.f, 0.f);
                        v[4 * x] = t.x * rkappa;
                        v[4 * x + 1] = t.y * rkappa;
                        v[4 * x + 2] = t.z * rkappa;
                        v[4 * x + 3] = t.w * rkappa;
                    }
                } else {
#pragma unroll
                    for (int x = 0; x < 16; ++x) v[x] = 0.f;
                    if (fr >= 0) v[0] = slot[D * DV + fr] * rkappa;
                }
                put_w(g, v, true);
            }
            w_ready();
        }

        for (int c = 0; c < nch && !bad; ++c) {
            const uint32_t cp = c & 1;
            if (c >= 1) {
                // W = gamma^C T from the carried state
                if (!mbar_wait(t_done, (c - 1) & 1, kErrMma)) { bad = true; break; }
                tc_fence_after();
                // the dv value columns in 16-column groups; the normaliser column
                // (dv) alone after them: its group's other 15 columns stay zero
                constexpr int NGT = DV / 16;
#pragma unroll 1
                for (int g0 = sub; g0 < NGT; g0 += KB * NTQ) {
                    float v[KB][16];
#pragma unroll
                    for (int i = 0; i < KB; ++i)
                        if (g0 + i * NTQ < NGT) tmem_ld16(tmem_addr(tbase, quad, P::T_T + (g0 + i * NTQ) * 16), v[i]);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < KB; ++i) tmem_regs_after_wait(v[i]);
#pragma unroll
                    for (int i = 0; i < KB; ++i)
                        if (g0 + i * NTQ < NGT) put_w(g0 + i * NTQ, v[i], DECAY);
                }
                if (sub == (DV / 16) % NTQ) {
                    float z = tmem_ld1(tmem_addr(tbase, quad, P::T_T + DV));
                    tmem_ld_wait();
                    tmem_regs_after_wait(z);
                    if (DECAY) {
                        z = one_factor ? z * gC : (z * gH) * gH;
                        tmem_st1(tmem_addr(tbase, quad, P::T_T + DV), z);
                    }
                    if (fr >= 0)
                        *reinterpret_cast<uint4*>(wcp + (DV / 64) * P::WBLK + sw128_offset(fr, 0)) =
                            make_uint4(pack_bf16x2(z, 0.f), 0u, 0u, 0u);
                }
                w_ready();
            }

            // P~ = causal mask of P (rows i); the previous chunk's MMA2 has read P~
            // (its output was waited for)
            if (!mbar_wait(p_full, cp, kErrMma)) { bad = true; break; }
            tc_fence_after();
            // This warp's rows are quad*16 .. quad*16+15 (lanes 0-15), so its column
            // groups below quad are kept whole, group quad is the diagonal block, and
            // the groups above are zero (not loaded).
#pragma unroll 1
            for (int g = sub; g < 4; g += NTQ) {
                uint32_t pk[8];
                if (g > quad) {
#pragma unroll
                    for (int h = 0; h < 8; ++h) pk[h] = 0u;
                } else {
                    float v[16];
                    tmem_ld16(tmem_addr(tbase, quad, P::T_P + g * 16), v);
                    tmem_ld_wait();
                    tmem_regs_after_wait(v);
                    if (g < quad) {
#pragma unroll
                        for (int h = 0; h < 8; ++h) pk[h] = pack_bf16x2(v[2 * h], v[2 * h + 1]);
                    } else {
#pragma unroll
                        for (int h = 0; h < 8; ++h) {
                            const int j = g * 16 + 2 * h;
                            pk[h] = pack_bf16x2(j <= ir ? v[2 * h] : 0.f, j + 1 <= ir ? v[2 * h + 1] : 0.f);
                        }
                    }
                }
                if (ir >= 0) {
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(ir, g * 32)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(ir, g * 32 + 16)) =
                        make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ptil_rdy);

            // output rows: o = O[:, :dv] / (O[:, dv] + eps) -> staging
            if (!mbar_wait(o_full, cp, kErrMma)) { bad = true; break; }
            tc_fence_after();
            float den = tmem_ld1(tmem_addr(tbase, quad, P::T_O + DV));
            if (c >= 1 && !mbar_wait(os_empty, (c - 1) & 1, kErrMma)) bad = true;
            const bool direct = clip_tail && c == nch - 1;
            const int nrow = chunk_len(c);
            constexpr int NGO = DV / 16;
            // up to four 16-column groups per wait: the output step is bound by the
            // TMEM load round trip (four per wait measured 7 % faster on the decay
            // workload than one)
            constexpr int KBO = (NGO + NTQ - 1) / NTQ < 4 ? (NGO + NTQ - 1) / NTQ : 4;
#pragma unroll 1
            for (int g0 = sub; g0 < NGO; g0 += KBO * NTQ) {
                float v[KBO][16];
#pragma unroll
                for (int i = 0; i < KBO; ++i)
                    if (g0 + i * NTQ < NGO) tmem_ld16(tmem_addr(tbase, quad, P::T_O + (g0 + i * NTQ) * 16), v[i]);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < KBO; ++i) tmem_regs_after_wait(v[i]);
                tmem_regs_after_wait(den);
                const float rden = __frcp_rn(den + eps);
#pragma unroll
                for (int i = 0; i < KBO; ++i) {
                    const int g = g0 + i * NTQ;
                    if (g < NGO) {
                    const float* o = v[i];
                    const uint4 lo = make_uint4(pack_bf16x2(o[0] * rden, o[1] * rden), pack_bf16x2(o[2] * rden, o[3] * rden),
                                                pack_bf16x2(o[4] * rden, o[5] * rden), pack_bf16x2(o[6] * rden, o[7] * rden));
                    const uint4 hi = make_uint4(pack_bf16x2(o[8] * rden, o[9] * rden), pack_bf16x2(o[10] * rden, o[11] * rden),
                                                pack_bf16x2(o[12] * rden, o[13] * rden),
                                                pack_bf16x2(o[14] * rden, o[15] * rden));
                    if (direct) {
                        // the padded batch's last rows of this sequence: only rows < n are written
                        if (ir >= 0 && ir < nrow) {
                            uint4* dst = reinterpret_cast<uint4*>(out + ((size_t)chain * ld + t0 + c * C + ir) * DV + g * 16);
                            dst[0] = lo;
                            dst[1] = hi;
                        }
                    } else if (ir >= 0) {
                        unsigned char* blk = otil + (g / 4) * TILE;
                        const int byte0 = (g % 4) * 32;
                        *reinterpret_cast<uint4*>(blk + sw128_offset(ir, byte0)) = lo;
                        *reinterpret_cast<uint4*>(blk + sw128_offset(ir, byte0 + 16)) = hi;
                    }
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
cudaError_t launch_tc_map(const PrefillArgs& a, const SegMap& m, int units)
{
    const int chains = a.B * a.H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, D, a.N, chains, a.ld) || !make_map(&mk, a.k, D, a.N, chains, a.ld) ||
        !make_map(&mv, a.v, DV, a.N, chains, a.ld) || !make_map(&mo, a.out, DV, a.N, chains, a.ld))
        return cudaErrorInvalidValue;
    float* ws = static_cast<float*>(a.workspace);

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
    lc.blockDim = dim3(kThreads + 32);   // + the issuing warp
    lc.dynamicSmemBytes = sa;
    lc.stream = a.stream;
    lc.attrs = pdl;
    lc.numAttrs = a.pdl_first ? 1 : 0;
    e = cudaLaunchKernelEx(&lc, ka, mk, mv, a.gamma, ws, m);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(0, a.stream);

    lc.gridDim = dim3(chains, kScanSplit);
    lc.blockDim = dim3(kScanThreads);
    lc.dynamicSmemBytes = 0;
    lc.numAttrs = 1;
    e = cudaLaunchKernelEx(&lc, scan_kernel<D, DV, DECAY>, ws, a.gamma, a.S0, a.z0, a.S_out, a.z_out, m);
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
    lc.blockDim = dim3(ChunkPlan<D, DV, DECAY>::THREADS);
    lc.dynamicSmemBytes = sc;
    e = cudaLaunchKernelEx(&lc, kc, mq, mk, mv, mo, a.gamma, (const float*)ws, m, a.eps,
                           static_cast<__nv_bfloat16*>(a.out), a.ld);
    if (e != cudaSuccess) return e;
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(2, a.stream);
    return cudaSuccess;
}

template <int D, int DV, bool DECAY>
cudaError_t launch_tc(const PrefillArgs& a, const TcSegments& sg)
{
    SegMap m;
    m.H = a.H;
    m.L = sg.L;
    m.B = 0;
    m.N = a.N;
    m.G = sg.G;
    return launch_tc_map<D, DV, DECAY>(a, m, a.B * a.H * sg.G);
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

// A right-padded batch as one launch set: one segment length L for all
// sequences, the smallest multiple of the chunk (at least two chunks) whose
// units fit one wave of resident CTAs, at most 4096 tokens.
namespace {
long long varlen_units(const int* lens, int B, int H, int L)
{
    long long u = 0;
    for (int b = 0; b < B; ++b) u += (long long)H * ((lens[b] + L - 1) / L);
    return u;
}
}  // namespace

int varlen_segment_length(const int* lens, int B, int H, int d, int dv)
{
    const long long slots = (d == 64 && dv == 64) ? 2 * 148 : 148;
    int L = 2 * C;
    while (L < 4096 && varlen_units(lens, B, H, L) > slots) L += C;
    return L;
}

size_t tc_varlen_workspace_bytes(const int* lens, int B, int H, int d, int dv)
{
    const int L = varlen_segment_length(lens, B, H, d, dv);
    return (size_t)varlen_units(lens, B, H, L) * ((size_t)d * dv + d) * sizeof(float);
}

cudaError_t launch_prefill_tc_kernelized_varlen(const PrefillArgs& a, const int* lens)
{
    if (a.B > kMaxVarlenSeqs) return cudaErrorInvalidValue;
    SegMap m;
    m.H = a.H;
    m.L = varlen_segment_length(lens, a.B, a.H, a.d, a.dv);
    m.B = a.B;
    for (int b = 0; b < a.B; ++b) m.lens[b] = lens[b];
    const long long units = varlen_units(lens, a.B, a.H, m.L);
    if (!a.workspace || a.workspace_bytes < tc_varlen_workspace_bytes(lens, a.B, a.H, a.d, a.dv))
        return cudaErrorInvalidValue;
    if (units == 0 || units > 0x7fffffffLL) return cudaErrorInvalidValue;
    const bool dec = a.mode == LA_DECAY;
#define LA_TC(D, DV)                                                                                   \
    if (a.d == D && a.dv == DV)                                                                         \
        return dec ? launch_tc_map<D, DV, true>(a, m, (int)units) : launch_tc_map<D, DV, false>(a, m, (int)units);
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
