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
#include <cudaTypedefs.h>

#include <mutex>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"
#include "sm100.cuh"

namespace la {
namespace {

using namespace sm100;

constexpr int C = 64;            // tokens per chunk
constexpr int kThreads = 128;    // one warpgroup: TMEM lanes 0..127
constexpr int TILE = C * 64 * 2; // one 64-token x 64-element bf16 tile (8 KB)

// ---------------------------------------------------------------------------
// Shared-memory plan of the chunk kernel (all tiles 1024-byte aligned).
template <int D, int DV, bool DECAY>
struct ChunkPlan {
    static constexpr int STAGES = (D + DV > 128) ? 3 : 4;
    static constexpr int QB = C * D * 2, KB = C * D * 2, VB = C * DV * 2;
    static constexpr int STAGE = QB + KB + VB;
    static constexpr int OFF_KT = STAGES * STAGE;
    static constexpr int OFF_P = OFF_KT + (DECAY ? KB : 0);
    static constexpr int OFF_SB = OFF_P + C * C * 2;
    static constexpr int OFF_O = OFF_SB + D * DV * 2;
    static constexpr int OFF_MISC = OFF_O + C * DV * 2;
    // misc: rden[C], qsc[C], dtab[C], z[2][D], barriers, tmem base
    static constexpr int OFF_RDEN = OFF_MISC;
    static constexpr int OFF_QSC = OFF_RDEN + C * 4;
    static constexpr int OFF_DTAB = OFF_QSC + C * 4;
    static constexpr int OFF_Z = OFF_DTAB + C * 4;
    static constexpr int OFF_BAR = OFF_Z + 2 * D * 4;
    static constexpr int NBAR = STAGES + 3;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;  // + alignment slack
    // TMEM columns
    static constexpr uint32_t T_P = 0, T_O = 64, T_OI = 128, T_S = 256, T_COLS = 512;
};

template <int D, int DV>
struct SummaryPlan {
    static constexpr int STAGES = 4;
    static constexpr int KB = C * D * 2, VB = C * DV * 2;
    static constexpr int STAGE = KB + VB;
    static constexpr int OFF_BAR = STAGES * STAGE;          // full[S], empty[S], done
    static constexpr int OFF_TMEM = OFF_BAR + (2 * STAGES + 1) * 8;
    static constexpr int BYTES = OFF_TMEM + 16 + 1024;
    static constexpr uint32_t T_COLS = DV < 32 ? 32 : DV;
};

__device__ __forceinline__ unsigned char* align1024(unsigned char* p)
{
    return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Row of an accumulator that this thread owns after tcgen05.ld.32x32b, for a
// tile of M rows (M = 128: lane i = row i; M = 64: rows 16w..16w+15 live in
// lanes 32w..32w+15).  Returns -1 when the lane holds no row.
template <int M>
__device__ __forceinline__ int acc_row(int warp, int lane)
{
    if (M == 128) return warp * 32 + lane;
    return lane < 16 ? warp * 16 + lane : -1;
}

__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, int warp, uint32_t col)
{
    return base + ((uint32_t)(warp * 32) << 16) + col;
}

// phi on a 16-byte chunk of 8 bf16 values, scaled by w; returns the packed chunk.
__device__ __forceinline__ uint4 phi_chunk(uint4 x, float w)
{
    uint32_t in[4] = {x.x, x.y, x.z, x.w};
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&in[i]);
        const float2 f = __bfloat1622float2(h);
        out[i] = pack_bf16x2(w * phi_fast(f.x), w * phi_fast(f.y));
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// ---------------------------------------------------------------------------
// Kernel A: segment summaries  Delta S = sum_t gamma^(last-t) phi(k_t) v_t^T,
// Delta z = sum_t gamma^(last-t) phi(k_t), over the tokens of one segment.
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kThreads, 1)
summary_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const float* __restrict__ gamma, float* __restrict__ ws, int N, int H, int G, int L)
{
    using P = SummaryPlan<D, DV>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* empty = full + P::STAGES;
    uint64_t* done = empty + P::STAGES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const float lam = DECAY ? logf(gamma[chain % H]) : 0.f;
    const uint64_t pol = policy_evict_normal();

    if (tid == 0) {
        for (int s = 0; s < P::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
        mbar_init(done, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    auto issue = [&](int c) {
        const int s = c % P::STAGES;
        unsigned char* st = sm + s * P::STAGE;
        mbar_expect_tx(&full[s], P::STAGE);
        for (int b = 0; b < D / 64; ++b) tma_load_3d(st + b * TILE, &tm_k, b * 64, t0 + c * C, chain, &full[s], pol);
        for (int b = 0; b < DV / 64; ++b)
            tma_load_3d(st + P::KB + b * TILE, &tm_v, b * 64, t0 + c * C, chain, &full[s], pol);
    };
    if (tid == 0)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);

    bool bad = false;
    float zacc = 0.f;
    const int last = t1 - 1;
    for (int c = 0; c < nch; ++c) {
        const int s = c % P::STAGES;
        const uint32_t ph = (c / P::STAGES) & 1;
        unsigned char* kt = sm + s * P::STAGE;
        unsigned char* vt = kt + P::KB;
        if (!mbar_wait(&full[s], ph, kErrTmaLoad)) bad = true;
        // K~_t = gamma^(last - t) phi(k_t), zero past the end of the sequence
        const int tc0 = t0 + c * C;
        for (int e = tid; e < (D / 8) * C; e += kThreads) {
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            uint4* p = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
            const int t = tc0 + row;
            const float w = t <= last ? (DECAY ? __expf((float)(last - t) * lam) : 1.f) : 0.f;
            *p = phi_chunk(*p, w);
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
        if (tid == 0) {
            tc_fence_after();
            const uint32_t idesc = idesc_bf16_f32(D, DV, 1, 1);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                const uint64_t a = sdesc_sw128(smem_u32(kt) + ks * 2048, TILE, 1024);
                const uint64_t bb = sdesc_sw128(smem_u32(vt) + ks * 2048, TILE, 1024);
                mma_bf16(tbase, a, bb, idesc, (c > 0 || ks > 0) ? 1u : 0u);
            }
            mma_commit(&empty[s]);
            if (c == nch - 1) mma_commit(done);
        }
        // Delta z: column sums of the bf16 K~ the tensor core consumes
        if (tid < D) {
            const int b = tid / 64, col = tid % 64;
            const unsigned char* base = kt + b * TILE;
            float acc = 0.f;
#pragma unroll 8
            for (int r = 0; r < C; ++r)
                acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + sw128_offset(r, col * 2)));
            zacc += acc;
        }
        // refill this stage once every thread is done with it and the MMA has consumed it
        __syncthreads();
        if (tid == 0 && c + P::STAGES < nch) {
            if (!mbar_wait(&empty[s], ph, kErrMma)) bad = true;
            else issue(c + P::STAGES);
        }
    }
    if (!bad && !mbar_wait(done, 0, kErrMma)) bad = true;
    tc_fence_after();
    float* slot = ws + (size_t)unit * (D * DV + D);
    if (!bad) {
        const int f = acc_row<D>(warp, lane);
#pragma unroll
        for (int g = 0; g < DV / 16; ++g) {
            float v[16];
            tmem_ld16(tmem_addr(tbase, warp, g * 16), v);
            tmem_ld_wait();
            if (f >= 0) {
                float4* dst = reinterpret_cast<float4*>(slot + (size_t)f * DV + g * 16);
#pragma unroll
                for (int q = 0; q < 4; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
            }
        }
        if (tid < D) slot[D * DV + tid] = zacc;
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, P::T_COLS);
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
template <int D, int DV, bool DECAY>
__global__ void __launch_bounds__(kThreads, 1)
chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
             const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
             const float* __restrict__ gamma, const float* __restrict__ ws, int N, int H, int G, int L, float eps)
{
    using P = ChunkPlan<D, DV, DECAY>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* sm = align1024(smem_raw);
    unsigned char* ktil = sm + P::OFF_KT;
    unsigned char* ptil = sm + P::OFF_P;
    unsigned char* sbt = sm + P::OFF_SB;
    unsigned char* otil = sm + P::OFF_O;
    float* rden = reinterpret_cast<float*>(sm + P::OFF_RDEN);
    float* qsc = reinterpret_cast<float*>(sm + P::OFF_QSC);
    float* dtab = reinterpret_cast<float*>(sm + P::OFF_DTAB);
    float* zbuf = reinterpret_cast<float*>(sm + P::OFF_Z);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + P::OFF_BAR);
    uint64_t* bar_p = full + P::STAGES;
    uint64_t* bar_s = bar_p + 1;
    uint64_t* bar_o = bar_p + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + P::OFF_TMEM);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int unit = blockIdx.x;
    const int chain = unit / G, seg = unit % G;
    const int t0 = seg * L, t1 = min(N, t0 + L);
    const int nch = (t1 - t0 + C - 1) / C;
    const float lam = DECAY ? logf(gamma[chain % H]) : 0.f;
    const uint64_t pol_in = policy_evict_first();

    if (tid == 0) {
        for (int s = 0; s < P::NBAR; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, P::T_COLS);
    if (tid < C) {
        dtab[tid] = DECAY ? __expf((float)tid * lam) : 1.f;        // gamma^(i-j)
        qsc[tid] = DECAY ? __expf((float)(tid + 1) * lam) : 1.f;    // gamma^(i+1)
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;

    // bookkeeping for the error path (meaningful in thread 0, which issues)
    int loads_issued = 0, loads_waited = 0, commits = 0, commits_o = 0;
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
    if (tid == 0)
        for (int c = 0; c < min(nch, P::STAGES); ++c) issue(c);

    // Start state: fp32 into TMEM (pre-scaled by gamma^n of the first chunk,
    // ready for MMA4 to accumulate onto), bf16 copy into smem for MMA3.
    {
        const float* slot = ws + (size_t)unit * (D * DV + D);
        const int f = acc_row<D>(warp, lane);
        const float dec0 = DECAY ? __expf((float)chunk_len(0) * lam) : 1.f;
#pragma unroll
        for (int g = 0; g < DV / 16; ++g) {
            float v[16];
            if (f >= 0) {
                const float4* src = reinterpret_cast<const float4*>(slot + (size_t)f * DV + g * 16);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 x = src[q];
                    v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
                }
                uint4 c0, c1;
                c0.x = pack_bf16x2(v[0], v[1]); c0.y = pack_bf16x2(v[2], v[3]);
                c0.z = pack_bf16x2(v[4], v[5]); c0.w = pack_bf16x2(v[6], v[7]);
                c1.x = pack_bf16x2(v[8], v[9]); c1.y = pack_bf16x2(v[10], v[11]);
                c1.z = pack_bf16x2(v[12], v[13]); c1.w = pack_bf16x2(v[14], v[15]);
                unsigned char* blk = sbt + (g / 4) * (D * 128);
                *reinterpret_cast<uint4*>(blk + sw128_offset(f, (g % 4) * 32)) = c0;
                *reinterpret_cast<uint4*>(blk + sw128_offset(f, (g % 4) * 32 + 16)) = c1;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] *= dec0;
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = 0.f;
            }
            tmem_st16(tmem_addr(tbase, warp, P::T_S + g * 16), v);
        }
        tmem_st_wait();
        if (tid < D) zbuf[tid] = slot[D * DV + tid];
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    bool bad = false;
    for (int c = 0; c < nch; ++c) {
        const int s = c % P::STAGES;
        const uint32_t ph = (c / P::STAGES) & 1;
        const uint32_t cp = c & 1;
        const int n = chunk_len(c);
        unsigned char* qt = sm + s * P::STAGE;
        unsigned char* kt = qt + P::QB;
        unsigned char* vt = kt + P::KB;
        unsigned char* kst = DECAY ? ktil : kt;   // K~ used by MMA4 and for z
        const float* zc = zbuf + cp * D;
        float* zn = zbuf + (cp ^ 1) * D;

        // 1. inputs landed; phi on load (K~ zeroed past the end of the sequence)
        if (!mbar_wait(&full[s], ph, kErrTmaLoad)) bad = true;
        else loads_waited = c + 1;
        for (int e = tid; e < (D / 8) * C; e += kThreads) {
            const int b = e / (8 * C), rem = e % (8 * C), row = rem / 8;
            uint4* pq = reinterpret_cast<uint4*>(qt + b * TILE) + rem;
            uint4* pk = reinterpret_cast<uint4*>(kt + b * TILE) + rem;
            *pq = phi_chunk(*pq, 1.f);
            const float valid = row < n ? 1.f : 0.f;
            const uint4 raw = *pk;
            *pk = phi_chunk(raw, valid);
            if (DECAY) {
                const float w = row < n ? __expf((float)(n - 1 - row) * lam) : 0.f;
                reinterpret_cast<uint4*>(ktil + b * TILE)[rem] = phi_chunk(raw, w);
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // 2. issue MMA1 (scores), MMA3 (start-state read), MMA4 (state carry)
        if (tid == 0) {
            tc_fence_after();
            const uint32_t qa = smem_u32(qt), ka = smem_u32(kt), va = smem_u32(vt);
            const uint32_t id1 = idesc_bf16_f32(64, 64, 0, 0);
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint32_t off = (ks / 4) * TILE + (ks % 4) * 32;
                mma_bf16(tbase + P::T_P, sdesc_sw128(qa + off, 16, 1024), sdesc_sw128(ka + off, 16, 1024), id1,
                         ks > 0);
            }
            mma_commit(bar_p);
            const uint32_t id3 = idesc_bf16_f32(DV, 64, 1, 0);
            const uint32_t oreg = DECAY ? P::T_OI : P::T_O;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                const uint64_t a = sdesc_sw128(smem_u32(sbt) + ks * 2048, D * 128, 1024);
                const uint64_t b = sdesc_sw128(qa + (ks / 4) * TILE + (ks % 4) * 32, 16, 1024);
                mma_bf16(tbase + oreg, a, b, id3, ks > 0);
            }
            const uint32_t id4 = idesc_bf16_f32(D, DV, 1, 1);
            const uint32_t kst_a = smem_u32(kst);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_S, sdesc_sw128(kst_a + ks * 2048, TILE, 1024),
                         sdesc_sw128(va + ks * 2048, TILE, 1024), id4, 1u);
            mma_commit(bar_s);
            commits = c + 1;
            // prefetch: the stage chunk c-1 used is free (its MMAs completed)
            if (c >= 1 && c - 1 + P::STAGES < nch) issue(c - 1 + P::STAGES);
        }

        // 3. scores -> P~ (mask, decay, bf16) and denominators
        if (!mbar_wait(bar_p, cp, kErrMma)) bad = true;
        tc_fence_after();
        {
            const int i = acc_row<64>(warp, lane);
            float praw[64];
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float v[16];
                tmem_ld16(tmem_addr(tbase, warp, P::T_P + g * 16), v);
#pragma unroll
                for (int x = 0; x < 16; ++x) praw[g * 16 + x] = v[x];
            }
            tmem_ld_wait();
            if (i >= 0) {
                float rs = 0.f;
#pragma unroll
                for (int cc = 0; cc < 8; ++cc) {
                    uint32_t pk[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int j0 = cc * 8 + 2 * h;
                        const float a = j0 <= i ? praw[j0] * dtab[i - j0] : 0.f;
                        const float b = j0 + 1 <= i ? praw[j0 + 1] * dtab[i - j0 - 1] : 0.f;
                        pk[h] = pack_bf16x2(a, b);
                        const float2 r = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[h]));
                        rs += r.x + r.y;
                    }
                    *reinterpret_cast<uint4*>(ptil + sw128_offset(i, cc * 16)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
                float qz = 0.f;
#pragma unroll
                for (int b = 0; b < D / 64; ++b)
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {
                        const uint4 x = *reinterpret_cast<const uint4*>(qt + b * TILE + sw128_offset(i, cc * 16));
                        const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                        for (int h = 0; h < 4; ++h) {
                            const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w4[h]));
                            const int fi = b * 64 + cc * 8 + 2 * h;
                            qz = fmaf(f.x, zc[fi], qz);
                            qz = fmaf(f.y, zc[fi + 1], qz);
                        }
                    }
                rden[i] = 1.f / (rs + qsc[i] * qz + eps);
            }
        }
        if (tid == 0) tma_store_wait_read();   // staging tile free again
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }

        // 4. MMA2: intra-chunk values
        if (tid == 0) {
            tc_fence_after();
            const uint32_t id2 = idesc_bf16_f32(DV, 64, 1, 0);
            const uint32_t va = smem_u32(vt), pa = smem_u32(ptil);
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks)
                mma_bf16(tbase + P::T_O, sdesc_sw128(va + ks * 2048, TILE, 1024),
                         sdesc_sw128(pa + ks * 32, 16, 1024), id2, (DECAY && ks == 0) ? 0u : 1u);
            mma_commit(bar_o);
            commits_o = c + 1;
        }

        // 5. state carry done: bf16 copy of S for the next chunk's MMA3,
        //    pre-scale for the next chunk's MMA4, normaliser update
        if (!mbar_wait(bar_s, cp, kErrMma)) bad = true;
        tc_fence_after();
        {
            const int f = acc_row<D>(warp, lane);
            const float decn = (DECAY && c + 1 < nch) ? __expf((float)chunk_len(c + 1) * lam) : 1.f;
#pragma unroll
            for (int g = 0; g < DV / 16; ++g) {
                float v[16];
                tmem_ld16(tmem_addr(tbase, warp, P::T_S + g * 16), v);
                tmem_ld_wait();
                if (f >= 0) {
                    uint4 c0, c1;
                    c0.x = pack_bf16x2(v[0], v[1]); c0.y = pack_bf16x2(v[2], v[3]);
                    c0.z = pack_bf16x2(v[4], v[5]); c0.w = pack_bf16x2(v[6], v[7]);
                    c1.x = pack_bf16x2(v[8], v[9]); c1.y = pack_bf16x2(v[10], v[11]);
                    c1.z = pack_bf16x2(v[12], v[13]); c1.w = pack_bf16x2(v[14], v[15]);
                    unsigned char* blk = sbt + (g / 4) * (D * 128);
                    *reinterpret_cast<uint4*>(blk + sw128_offset(f, (g % 4) * 32)) = c0;
                    *reinterpret_cast<uint4*>(blk + sw128_offset(f, (g % 4) * 32 + 16)) = c1;
                }
                if (DECAY) {
#pragma unroll
                    for (int x = 0; x < 16; ++x) v[x] *= decn;
                    tmem_st16(tmem_addr(tbase, warp, P::T_S + g * 16), v);
                }
            }
            if (DECAY) tmem_st_wait();
            if (tid < D) {
                const int b = tid / 64, col = tid % 64;
                const unsigned char* base = kst + b * TILE;
                float acc = 0.f;
#pragma unroll 8
                for (int r = 0; r < C; ++r)
                    acc += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(base + sw128_offset(r, col * 2)));
                const float dec = DECAY ? __expf((float)n * lam) : 1.f;
                zn[tid] = fmaf(dec, zc[tid], acc);
            }
        }
        fence_async_smem();

        // 6. outputs: o_i = (O_intra + gamma^(i+1) O_inter) / den_i -> staging -> TMA store
        if (!mbar_wait(bar_o, cp, kErrMma)) bad = true;
        tc_fence_after();
        {
            const int j = acc_row<DV>(warp, lane);
            unsigned char* oblk = otil + (j >= 0 ? (j / 64) * TILE : 0);
            const int jb = (j >= 0 ? (j % 64) : 0) * 2;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                float v[16], w[16];
                tmem_ld16(tmem_addr(tbase, warp, P::T_O + g * 16), v);
                if (DECAY) tmem_ld16(tmem_addr(tbase, warp, P::T_OI + g * 16), w);
                tmem_ld_wait();
                if (j >= 0) {
#pragma unroll
                    for (int x = 0; x < 16; ++x) {
                        const int i = g * 16 + x;
                        const float num = DECAY ? fmaf(qsc[i], w[x], v[x]) : v[x];
                        *reinterpret_cast<__nv_bfloat16*>(oblk + sw128_offset(i, jb)) =
                            __float2bfloat16_rn(num * rden[i]);
                    }
                }
            }
        }
        fence_async_smem();
        tc_fence_before();
        if (__syncthreads_or(bad)) { bad = true; break; }
        if (tid == 0) {
            for (int b = 0; b < DV / 64; ++b) tma_store_3d(&tm_o, otil + b * TILE, b * 64, t0 + c * C, chain);
            tma_store_commit();
        }
    }
    if (tid == 0) tma_store_wait_all();
    if (bad && tid == 0) {
        // Leave no copy or MMA in flight before releasing TMEM and exiting:
        // wait (bounded) for every issued load not yet consumed and for the
        // last commit of each MMA barrier.
        for (int cc = loads_waited; cc < loads_issued; ++cc)
            mbar_wait(&full[cc % P::STAGES], (cc / P::STAGES) & 1, kErrTmaLoad);
        if (commits > 0) {
            const uint32_t last = (commits - 1) & 1;
            mbar_wait(bar_p, last, kErrMma);
            mbar_wait(bar_s, last, kErrMma);
            if (commits_o > 0) mbar_wait(bar_o, (commits_o - 1) & 1, kErrMma);
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

// 3-D map over a bf16 [chains][N][inner] tensor; box = 64 elements x 64 rows,
// 128-byte swizzle; rows past N read as zero and are not written.
bool make_map(CUtensorMap* m, const void* base, int inner, int N, int chains)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)N, (cuuint64_t)chains};
    cuuint64_t strides[2] = {(cuuint64_t)inner * 2, (cuuint64_t)N * inner * 2};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int DV, bool DECAY>
cudaError_t launch_tc(const PrefillArgs& a, const TcSegments& sg)
{
    const int chains = a.B * a.H;
    CUtensorMap mq, mk, mv, mo;
    if (!make_map(&mq, a.q, D, a.N, chains) || !make_map(&mk, a.k, D, a.N, chains) ||
        !make_map(&mv, a.v, DV, a.N, chains) || !make_map(&mo, a.out, DV, a.N, chains))
        return cudaErrorInvalidValue;
    float* ws = static_cast<float*>(a.workspace);
    const int units = chains * sg.G;

    auto ka = summary_kernel<D, DV, DECAY>;
    const int sa = SummaryPlan<D, DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, sa);
    if (e != cudaSuccess) return e;
    ka<<<units, kThreads, sa, a.stream>>>(mk, mv, a.gamma, ws, a.N, a.H, sg.G, sg.L);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    constexpr int SLOT = D * DV + D;
    dim3 gs(chains, (SLOT + 255) / 256);
    scan_kernel<D, DV, DECAY><<<gs, 256, 0, a.stream>>>(ws, a.gamma, a.S0, a.z0, a.S_out, a.z_out, a.N, a.H,
                                                        sg.G, sg.L);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    auto kc = chunk_kernel<D, DV, DECAY>;
    const int sc = ChunkPlan<D, DV, DECAY>::BYTES;
    e = cudaFuncSetAttribute(kc, cudaFuncAttributeMaxDynamicSharedMemorySize, sc);
    if (e != cudaSuccess) return e;
    kc<<<units, kThreads, sc, a.stream>>>(mq, mk, mv, mo, a.gamma, ws, a.N, a.H, sg.G, sg.L, a.eps);
    return cudaGetLastError();
}

}  // namespace

TcSegments tc_segments(int B, int H, int N, int d, int dv)
{
    (void)d; (void)dv;
    TcSegments s;
    const long long chains = (long long)B * H;
    const long long target = 4LL * 148;  // about four CTAs per SM over the launch
    long long L = chains > 0 ? (N * chains + target - 1) / target : N;
    L = ((L + C - 1) / C) * C;
    if (L < 2 * C) L = 2 * C;
    s.L = (int)L;
    s.G = N > 0 ? (int)((N + L - 1) / L) : 0;
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
