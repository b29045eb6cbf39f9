// SIMT (CUDA-core, fp32 arithmetic) prefill kernels.
//
// These kernels carry the fp32-input path, where bf16 tensor-core operands
// could not meet a 1e-4 relative error, and they accept bf16 inputs as well.
//
// kernelized (LA_PLAIN / LA_DECAY): chunkwise form ("Efficient attention
// variants" §8).  For a chunk of C tokens with start state (S0, z0), local
// positions i, j = 0..C-1 and lambda = log gamma:
//   P_ij  = [j <= i] exp((i-j) lambda) phi(q_i).phi(k_j)     (multiplicative
//           causal + decay mask, "Transformers Are RNNs" notes)
//   num_i = sum_j P_ij v_j + exp((i+1) lambda) phi(q_i)^T S0
//   den_i = sum_j P_ij     + exp((i+1) lambda) phi(q_i)^T z0
//   o_i   = num_i / (den_i + eps)
//   S    <- exp(n lambda) S0 + sum_j exp((n-1-j) lambda) phi(k_j) v_j^T
//   z    <- exp(n lambda) z0 + sum_j exp((n-1-j) lambda) phi(k_j)
// with n the number of valid tokens in the chunk.  This is the unrolled
// recurrence S_t = gamma S_{t-1} + phi(k_t) v_t^T of "What Is Linear
// Attention?" §4/§5.1 regrouped by chunk; it is exact up to rounding order.
//
// gated delta (LA_GATED_DELTA): the token recurrence itself, one thread per
// state column.  Columns of S evolve independently under the delta rule
// (S^T k is a per-column dot product), so each thread keeps its column of S
// in registers: vhat_j = S_j.k_t;  S_j <- alpha S_j + g k_t (v_tj - alpha vhat_j);
// o_tj = S_j.q_t   ("Efficient attention variants" §7.4).
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kChunk = 32;   // tokens per chunk
constexpr int kThreads = 256;

template <int D, int DVT>
struct KernelizedSmem {
    float fq[kChunk][D + 1];
    float fk[kChunk][D + 1];
    float vv[kChunk][DVT];
    float P[kChunk][kChunk + 1];
    float S[D][DVT];
    float z[D];
    float den[kChunk];
    float wk[kChunk];  // exp((n-1-j) lambda)
};

template <typename T, int D, int DVT>
__global__ void __launch_bounds__(kThreads)
kernelized_chunk_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                      const float* __restrict__ gamma, const float* __restrict__ S0,
                      const float* __restrict__ z0, T* __restrict__ out, float* __restrict__ S_out,
                      float* __restrict__ z_out, int H, int N, int dv, float eps, int ld)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<KernelizedSmem<D, DVT>*>(smem_raw);
    const int tid = threadIdx.x;
    const int j0 = blockIdx.y * DVT;       // first value column of this tile
    const long long chain = blockIdx.x;    // b*H + h
    const int h = (int)(chain % H);
    const float lam = gamma ? logf(gamma[h]) : 0.f;

    const T* qc = q + chain * (long long)ld * D;
    const T* kc = k + chain * (long long)ld * D;
    const T* vc = v + chain * (long long)ld * dv;
    T* oc = out + chain * (long long)ld * dv;

    for (int e = tid; e < D * DVT; e += kThreads) {
        const int f = e / DVT, j = e % DVT;
        sm.S[f][j] = S0 ? S0[chain * (long long)D * dv + (long long)f * dv + j0 + j] : 0.f;
    }
    for (int f = tid; f < D; f += kThreads) sm.z[f] = z0 ? z0[chain * D + f] : 0.f;

    for (int c0 = 0; c0 < N; c0 += kChunk) {
        const int n = min(kChunk, N - c0);
        __syncthreads();  // previous chunk finished with every buffer
        for (int e = tid; e < kChunk * D; e += kThreads) {
            const int t = e / D, f = e % D;
            const bool ok = t < n;
            const long long off = (long long)(c0 + t) * D + f;
            sm.fq[t][f] = ok ? phi(to_f32(qc[off])) : 0.f;
            sm.fk[t][f] = ok ? phi(to_f32(kc[off])) : 0.f;
        }
        for (int e = tid; e < kChunk * DVT; e += kThreads) {
            const int t = e / DVT, j = e % DVT;
            sm.vv[t][j] = t < n ? to_f32(vc[(long long)(c0 + t) * dv + j0 + j]) : 0.f;
        }
        if (tid < kChunk) sm.wk[tid] = tid < n ? expf((float)(n - 1 - tid) * lam) : 0.f;
        __syncthreads();

        // P = (phi(Q) phi(K)^T) * mask * decay
        for (int e = tid; e < kChunk * kChunk; e += kThreads) {
            const int i = e / kChunk, j = e % kChunk;
            float s = 0.f;
            if (j <= i) {
#pragma unroll 8
                for (int f = 0; f < D; ++f) s = fmaf(sm.fq[i][f], sm.fk[j][f], s);
                s *= expf((float)(i - j) * lam);
            }
            sm.P[i][j] = s;
        }
        __syncthreads();

        // denominators: row sums of P plus the start-state term
        if (tid < kChunk) {
            const int i = tid;
            float r = 0.f;
            for (int j = 0; j <= i; ++j) r += sm.P[i][j];
            float qz = 0.f;
            for (int f = 0; f < D; ++f) qz = fmaf(sm.fq[i][f], sm.z[f], qz);
            sm.den[i] = r + expf((float)(i + 1) * lam) * qz + eps;
        }
        __syncthreads();

        // numerators and outputs
        for (int e = tid; e < kChunk * DVT; e += kThreads) {
            const int i = e / DVT, j = e % DVT;
            if (i >= n) continue;
            float intra = 0.f;
            for (int l = 0; l <= i; ++l) intra = fmaf(sm.P[i][l], sm.vv[l][j], intra);
            float inter = 0.f;
#pragma unroll 8
            for (int f = 0; f < D; ++f) inter = fmaf(sm.fq[i][f], sm.S[f][j], inter);
            const float num = intra + expf((float)(i + 1) * lam) * inter;
            oc[(long long)(c0 + i) * dv + j0 + j] = from_f32<T>(num / sm.den[i]);
        }
        __syncthreads();

        // state carry
        const float cdec = expf((float)n * lam);
        for (int e = tid; e < D * DVT; e += kThreads) {
            const int f = e / DVT, j = e % DVT;
            float s = 0.f;
            for (int l = 0; l < n; ++l) s = fmaf(sm.wk[l] * sm.fk[l][f], sm.vv[l][j], s);
            sm.S[f][j] = fmaf(cdec, sm.S[f][j], s);
        }
        for (int f = tid; f < D; f += kThreads) {
            float s = 0.f;
            for (int l = 0; l < n; ++l) s = fmaf(sm.wk[l], sm.fk[l][f], s);
            sm.z[f] = fmaf(cdec, sm.z[f], s);
        }
    }
    __syncthreads();
    for (int e = tid; e < D * DVT; e += kThreads) {
        const int f = e / DVT, j = e % DVT;
        S_out[chain * (long long)D * dv + (long long)f * dv + j0 + j] = sm.S[f][j];
    }
    if (blockIdx.y == 0)
        for (int f = tid; f < D; f += kThreads) z_out[chain * D + f] = sm.z[f];
}

template <typename T, int D, int DVT>
cudaError_t launch_kernelized_t(const PrefillArgs& a)
{
    auto kern = kernelized_chunk_simt<T, D, DVT>;
    const size_t smem = sizeof(KernelizedSmem<D, DVT>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.H, a.dv / DVT);
    kern<<<grid, kThreads, smem, a.stream>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, a.gamma, a.S0, a.z0,
                                             (T*)a.out, a.S_out, a.z_out, a.H, a.N, a.dv, a.eps, a.ld);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(0, a.stream);
    return cudaSuccess;
}

// ---------------------------------------------------------------------------
// gated delta, token recurrence, one thread per column of S.

constexpr int kDeltaTile = 32;  // tokens staged in shared memory at a time

template <typename T, int D>
__global__ void __launch_bounds__(128)
gated_delta_token_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ alpha, const float* __restrict__ g,
                       const float* __restrict__ S0, T* __restrict__ out, float* __restrict__ S_out,
                       int N, int dv, int ld)
{
    __shared__ __align__(16) float kq[2][kDeltaTile][D];
    __shared__ float ag[2][kDeltaTile];
    const int j = blockIdx.y * blockDim.x + threadIdx.x;  // state column
    const long long chain = blockIdx.x;
    const bool active = j < dv;
    const T* qc = q + chain * (long long)ld * D;
    const T* kc = k + chain * (long long)ld * D;
    const T* vc = v + chain * (long long)ld * dv;
    const float* al = alpha + chain * (long long)ld;
    const float* gl = g + chain * (long long)ld;
    T* oc = out + chain * (long long)ld * dv;

    float s[D];
#pragma unroll
    for (int i = 0; i < D; ++i)
        s[i] = (S0 && active) ? S0[chain * (long long)D * dv + (long long)i * dv + j] : 0.f;

    for (int t0 = 0; t0 < N; t0 += kDeltaTile) {
        const int n = min(kDeltaTile, N - t0);
        __syncthreads();
        for (int e = threadIdx.x; e < kDeltaTile * D; e += blockDim.x) {
            const int t = e / D, f = e % D;
            const long long off = (long long)(t0 + t) * D + f;
            kq[0][t][f] = t < n ? to_f32(kc[off]) : 0.f;
            kq[1][t][f] = t < n ? to_f32(qc[off]) : 0.f;
        }
        for (int t = threadIdx.x; t < kDeltaTile; t += blockDim.x) {
            ag[0][t] = t < n ? al[t0 + t] : 1.f;
            ag[1][t] = t < n ? gl[t0 + t] : 0.f;
        }
        __syncthreads();
        for (int t = 0; t < n; ++t) {
            const float vt = active ? to_f32(vc[(long long)(t0 + t) * dv + j]) : 0.f;
            const float at = ag[0][t], gt = ag[1][t];
            float h0 = 0.f, h1 = 0.f, h2 = 0.f, h3 = 0.f;
#pragma unroll
            for (int i = 0; i < D; i += 4) {
                h0 = fmaf(s[i + 0], kq[0][t][i + 0], h0);
                h1 = fmaf(s[i + 1], kq[0][t][i + 1], h1);
                h2 = fmaf(s[i + 2], kq[0][t][i + 2], h2);
                h3 = fmaf(s[i + 3], kq[0][t][i + 3], h3);
            }
            const float vhat = (h0 + h1) + (h2 + h3);        // S_{t-1}^T k_t
            const float err = gt * (vt - at * vhat);          // g (v - alpha vhat)
            float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
#pragma unroll
            for (int i = 0; i < D; i += 4) {
                s[i + 0] = fmaf(at, s[i + 0], kq[0][t][i + 0] * err);
                s[i + 1] = fmaf(at, s[i + 1], kq[0][t][i + 1] * err);
                s[i + 2] = fmaf(at, s[i + 2], kq[0][t][i + 2] * err);
                s[i + 3] = fmaf(at, s[i + 3], kq[0][t][i + 3] * err);
                o0 = fmaf(s[i + 0], kq[1][t][i + 0], o0);
                o1 = fmaf(s[i + 1], kq[1][t][i + 1], o1);
                o2 = fmaf(s[i + 2], kq[1][t][i + 2], o2);
                o3 = fmaf(s[i + 3], kq[1][t][i + 3], o3);
            }
            if (active) oc[(long long)(t0 + t) * dv + j] = from_f32<T>((o0 + o1) + (o2 + o3));
        }
    }
    if (active) {
#pragma unroll
        for (int i = 0; i < D; ++i) S_out[chain * (long long)D * dv + (long long)i * dv + j] = s[i];
    }
}

template <typename T, int D>
cudaError_t launch_gdelta_t(const PrefillArgs& a)
{
    const int threads = 64;
    dim3 grid(a.B * a.H, (a.dv + threads - 1) / threads);
    gated_delta_token_simt<T, D><<<grid, threads, 0, a.stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, a.alpha, a.g, a.S0, (T*)a.out, a.S_out, a.N, a.dv, a.ld);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) stage_mark(0, a.stream);
    return e;
}

// ---------------------------------------------------------------------------
// GLA, per-key-channel gate ("Efficient attention variants" §7.2), token
// recurrence:
//     S_t[i][j] = alpha_t[i] S_{t-1}[i][j] + k_t[i] v_t[j],  o_t[j] = sum_i q_t[i] S_t[i][j]
// Eight threads share a state column, each holding a contiguous block of
// R = d/8 rows in registers, and add their parts of o_t with three shuffles.
// Per tile of kGlaTile tokens, k, q, alpha and the block's v columns stream
// into shared memory by cp.async (double-buffered); k and q are converted to
// fp32 once per tile, so the token loop reads every operand with 128-bit
// loads.  The fp32 rows are stored as 8 blocks of R values with a 16-byte
// skew between blocks (block stride an odd number of 16-byte units), so the
// eight row blocks a warp reads at once fall in distinct banks.  Outputs of a
// tile are collected in shared memory and written as 16-byte pieces.

constexpr int kGlaTile = 16;   // tokens per staged tile
constexpr int kGlaCols = 32;   // state columns per block
constexpr int kGlaTpc = 8;     // threads per state column
constexpr int kGlaThreads = kGlaCols * kGlaTpc;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, uint32_t src_bytes)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int Nleft>
__device__ __forceinline__ void cp_async_wait_groups() { asm volatile("cp.async.wait_group %0;" ::"n"(Nleft) : "memory"); }

template <typename T, int D>
struct GlaSmem {
    static constexpr int R = D / kGlaTpc;     // rows per thread
    static constexpr int BS = R + 4;          // fp32 row-block stride (R/4 + 1 16-byte units: odd)
    static constexpr int RS = kGlaTpc * BS;   // fp32 row stride
    T kr[2][kGlaTile][D];                     // k, q as loaded
    T qr[2][kGlaTile][D];
    float a[2][kGlaTile][RS];                 // alpha, skewed row blocks
    T v[2][kGlaTile][kGlaCols];
    float kf[kGlaTile][RS];                   // k, q in fp32, skewed row blocks
    float qf[kGlaTile][RS];
    float o[kGlaTile][kGlaCols];
};

template <typename T> __device__ __forceinline__ void unpack16(const uint4& u, float* f);
template <> __device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& u, float* f)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
template <> __device__ __forceinline__ void unpack16<float>(const uint4& u, float* f)
{
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
}

template <typename T, int D>
__global__ void __launch_bounds__(kGlaThreads)
gla_token_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
               const float* __restrict__ alpha, const float* __restrict__ S0, T* __restrict__ out,
               float* __restrict__ S_out, int N, int dv, int ld)
{
    using SM = GlaSmem<T, D>;
    constexpr int R = SM::R, BS = SM::BS;
    constexpr int EP = 16 / (int)sizeof(T);           // elements per 16-byte piece
    extern __shared__ __align__(16) unsigned char gla_smem[];
    SM& sh = *reinterpret_cast<SM*>(gla_smem);
    const int tid = threadIdx.x;
    const int rg = tid & (kGlaTpc - 1), jl = tid / kGlaTpc;   // row block, local column
    const int j = blockIdx.y * kGlaCols + jl;                 // state column
    const long long chain = blockIdx.x;
    const bool active = j < dv;
    const T* qc = q + chain * (long long)ld * D;
    const T* kc = k + chain * (long long)ld * D;
    const float* ac = alpha + chain * (long long)ld * D;
    const T* vc = v + chain * (long long)ld * dv + blockIdx.y * kGlaCols;
    T* oc = out + chain * (long long)ld * dv + blockIdx.y * kGlaCols;
    const int vcols = min(kGlaCols, dv - (int)blockIdx.y * kGlaCols);

    // this thread's rows: rg*R .. rg*R + R-1
    float s[R];
#pragma unroll
    for (int i = 0; i < R; ++i)
        s[i] = (S0 && active) ? S0[chain * (long long)D * dv + (long long)(rg * R + i) * dv + j] : 0.f;

    // stage tile `tile` into buffer `b`: 16-byte pieces, zero past the end
    auto stage = [&](int tile, int b) {
        const int t0 = tile * kGlaTile;
        constexpr int PR = D / EP;                              // pieces per k/q row
        constexpr int KQ = kGlaTile * PR;                       // pieces of k (and of q)
        constexpr int PA = D / 4;                               // pieces per alpha row
        constexpr int AP = kGlaTile * PA;
        constexpr int PV = kGlaCols / EP;                       // pieces per v row
        constexpr int VP = kGlaTile * PV;
        for (int e = tid; e < 2 * KQ + AP + VP; e += kGlaThreads) {
            if (e < 2 * KQ) {
                const int which = e / KQ, r = (e % KQ) / PR, c = (e % KQ) % PR;
                const int t = t0 + r;
                const T* src = (which ? qc : kc) + (long long)min(t, N - 1) * D + c * EP;
                T* dst = (which ? &sh.qr[b][r][0] : &sh.kr[b][r][0]) + c * EP;
                cp_async16(dst, src, t < N ? 16u : 0u);
            } else if (e < 2 * KQ + AP) {
                const int f = e - 2 * KQ, r = f / PA, f0 = (f % PA) * 4, t = t0 + r;
                cp_async16(&sh.a[b][r][(f0 / R) * BS + f0 % R], ac + (long long)min(t, N - 1) * D + f0,
                           t < N ? 16u : 0u);
            } else {
                const int f = e - 2 * KQ - AP, r = f / PV, col = (f % PV) * EP, t = t0 + r;
                const bool ok = t < N && col < vcols;
                cp_async16(&sh.v[b][r][col], vc + (long long)min(t, N - 1) * dv + (ok ? col : 0), ok ? 16u : 0u);
            }
        }
        cp_async_commit_group();
    };

    const int tiles = (N + kGlaTile - 1) / kGlaTile;
    stage(0, 0);
    for (int tile = 0; tile < tiles; ++tile) {
        const int b = tile & 1;
        if (tile + 1 < tiles) {
            stage(tile + 1, b ^ 1);
            cp_async_wait_groups<1>();
        } else {
            cp_async_wait_groups<0>();
        }
        __syncthreads();
        // k, q of this tile to fp32 (8 consecutive features stay in one row block)
        for (int e = tid; e < 2 * kGlaTile * (D / 8); e += kGlaThreads) {
            const int which = e / (kGlaTile * (D / 8)), rem = e % (kGlaTile * (D / 8));
            const int r = rem / (D / 8), f0 = (rem % (D / 8)) * 8;
            const T* src = (which ? &sh.qr[b][r][0] : &sh.kr[b][r][0]) + f0;
            float f[8];
            unpack16<T>(*reinterpret_cast<const uint4*>(src), f);
            if (EP == 4) unpack16<T>(*reinterpret_cast<const uint4*>(src + 4), f + 4);
            float* dst = (which ? &sh.qf[r][0] : &sh.kf[r][0]) + (f0 / R) * BS + f0 % R;
            reinterpret_cast<float4*>(dst)[0] = make_float4(f[0], f[1], f[2], f[3]);
            reinterpret_cast<float4*>(dst)[1] = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        const int n = min(kGlaTile, N - tile * kGlaTile);
        for (int t = 0; t < n; ++t) {
            const float vt = to_f32(sh.v[b][t][jl]);
            const float4* ap = reinterpret_cast<const float4*>(&sh.a[b][t][rg * BS]);
            const float4* kp = reinterpret_cast<const float4*>(&sh.kf[t][rg * BS]);
            const float4* qp = reinterpret_cast<const float4*>(&sh.qf[t][rg * BS]);
            float o0 = 0.f, o1 = 0.f;
#pragma unroll
            for (int i4 = 0; i4 < R / 4; ++i4) {
                const float4 a4 = ap[i4], k4 = kp[i4], q4 = qp[i4];
                float* si = s + 4 * i4;
                si[0] = fmaf(a4.x, si[0], k4.x * vt);
                si[1] = fmaf(a4.y, si[1], k4.y * vt);
                si[2] = fmaf(a4.z, si[2], k4.z * vt);
                si[3] = fmaf(a4.w, si[3], k4.w * vt);
                o0 = fmaf(si[0], q4.x, o0);
                o1 = fmaf(si[1], q4.y, o1);
                o0 = fmaf(si[2], q4.z, o0);
                o1 = fmaf(si[3], q4.w, o1);
            }
            float o = o0 + o1;
            o += __shfl_xor_sync(0xffffffffu, o, 1);
            o += __shfl_xor_sync(0xffffffffu, o, 2);
            o += __shfl_xor_sync(0xffffffffu, o, 4);
            if (rg == 0) sh.o[t][jl] = o;
        }
        __syncthreads();
        // this tile's outputs: n rows of the block's columns, 16-byte pieces
        {
            constexpr int PO = kGlaCols / EP;   // pieces per output row
            for (int e = tid; e < n * PO; e += kGlaThreads) {
                const int r = e / PO, col = (e % PO) * EP;
                if (col < vcols) {
                    const float* src = &sh.o[r][col];
                    T* dst = oc + (long long)(tile * kGlaTile + r) * dv + col;
                    if (EP == 8) {
                        uint32_t w[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const __nv_bfloat162 h = __floats2bfloat162_rn(src[2 * x], src[2 * x + 1]);
                            w[x] = *reinterpret_cast<const uint32_t*>(&h);
                        }
                        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
                    } else {
                        *reinterpret_cast<float4*>(dst) = *reinterpret_cast<const float4*>(src);
                    }
                }
            }
        }
    }
    if (active) {
#pragma unroll
        for (int i = 0; i < R; ++i) S_out[chain * (long long)D * dv + (long long)(rg * R + i) * dv + j] = s[i];
    }
}

template <typename T, int D>
cudaError_t launch_gla_t(const PrefillArgs& a)
{
    auto kern = gla_token_simt<T, D>;
    const int smem = (int)sizeof(GlaSmem<T, D>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dim3 grid(a.B * a.H, (a.dv + kGlaCols - 1) / kGlaCols);
    kern<<<grid, kGlaThreads, smem, a.stream>>>((const T*)a.q, (const T*)a.k, (const T*)a.v, a.alpha, a.S0,
                                                 (T*)a.out, a.S_out, a.N, a.dv, a.ld);
    e = cudaGetLastError();
    if (e == cudaSuccess) stage_mark(0, a.stream);
    return e;
}

// ---------------------------------------------------------------------------
// Short sequences (N <= kParallelMaxN): the parallel form of the same
// quantities, no chunk loop.  "What Is Linear Attention?" §3 and "Transformers
// Are RNNs" (the masked-matrix form equals the recurrence): for every token i
//   num_i = sum_{j <= i} gamma^(i-j) phi(q_i).phi(k_j) v_j + gamma^(i+1) phi(q_i)^T S0
//   den_i = sum_{j <= i} gamma^(i-j) phi(q_i).phi(k_j)     + gamma^(i+1) phi(q_i)^T z0
//   o_i   = num_i / (den_i + eps)
// and the final state
//   S_N = gamma^N S0 + sum_t gamma^(N-1-t) phi(k_t) v_t^T,   z_N likewise.
// Every output row and every state element is an independent sum, so a
// single short chain spreads over many CTAs instead of running its chunks
// one after another on one.

constexpr int kParallelMaxN = 1024;
constexpr int kRows = 16;    // query rows per CTA
constexpr int kKeys = 32;    // keys per staged block

// Row blocks of fp32 [rows][W] in 16-byte pieces, in two halves so that the
// loads of the next block are in flight while the current one is used: load()
// issues a thread's loads into registers, store() writes them to shared memory
// (row pitch P floats), phi applied when PHI, rows past nvalid as zeros.
template <int ROWS, int W>
struct RowBlock {
    static constexpr int V = ROWS * W / 4;                  // float4 pieces
    static constexpr int PER = (V + kThreads - 1) / kThreads;
    float4 x[PER];
    __device__ __forceinline__ void load(const float* __restrict__ src, int nvalid, int tid)
    {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * kThreads;
            const int row = e / (W / 4), c4 = e % (W / 4);
            x[u] = (e < V && row < nvalid) ? reinterpret_cast<const float4*>(src + (size_t)row * W)[c4]
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    template <int P, bool PHI>
    __device__ __forceinline__ void store(float (*sm)[P], int nvalid, int tid) const
    {
#pragma unroll
        for (int u = 0; u < PER; ++u) {
            const int e = tid + u * kThreads;
            if (e >= V) break;
            const int row = e / (W / 4), c = (e % (W / 4)) * 4;
            const bool ph = PHI && row < nvalid;
            sm[row][c] = ph ? phi(x[u].x) : x[u].x;
            sm[row][c + 1] = ph ? phi(x[u].y) : x[u].y;
            sm[row][c + 2] = ph ? phi(x[u].z) : x[u].z;
            sm[row][c + 3] = ph ? phi(x[u].w) : x[u].w;
        }
    }
};

template <int D, int DV>
struct ParallelSmem {
    float fq[kRows][D + 1];
    float fk[kKeys][D + 1];
    float vv[kKeys][DV];
    float P[kRows][kKeys + 1];
};

// grid (chains, ceil(N / kRows)), 256 threads: thread (r, c) accumulates row r,
// columns c, c + 16, ... of the numerator; every thread of a row keeps its den.
template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads)
kernelized_parallel_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const float* __restrict__ gamma, const float* __restrict__ S0,
                         const float* __restrict__ z0, T* __restrict__ out, int H, int N, float eps, int ld)
{
    static_assert(sizeof(T) == 4, "the parallel form stages fp32 rows");
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<ParallelSmem<D, DV>*>(smem_raw);
    constexpr int CPT = DV / 16;    // numerator columns per thread
    const int tid = threadIdx.x, r = tid / 16, cl = tid % 16;
    const long long chain = blockIdx.x;
    const int h = (int)(chain % H);
    const float lam = gamma ? logf(gamma[h]) : 0.f;
    const int i0 = blockIdx.y * kRows;
    const int rows = min(kRows, N - i0);
    const T* qc = q + chain * (long long)ld * D;
    const T* kc = k + chain * (long long)ld * D;
    const T* vc = v + chain * (long long)ld * DV;
    T* oc = out + chain * (long long)ld * DV;

    const float* kf = reinterpret_cast<const float*>(kc);
    const float* vf = reinterpret_cast<const float*>(vc);
    {
        RowBlock<kRows, D> qb;
        qb.load(reinterpret_cast<const float*>(qc) + (size_t)i0 * D, rows, tid);
        qb.store<D + 1, true>(sm.fq, rows, tid);
    }
    float num[CPT];
#pragma unroll
    for (int m = 0; m < CPT; ++m) num[m] = 0.f;
    float den = 0.f;
    const int i = i0 + r;
    const int jend = i0 + rows;    // keys 0 .. jend-1 reach some row of this CTA
    RowBlock<kKeys, D> kb;
    RowBlock<kKeys, DV> vb;
    kb.load(kf, min(kKeys, jend), tid);
    vb.load(vf, min(kKeys, jend), tid);
    for (int j0 = 0; j0 < jend; j0 += kKeys) {
        const int nk = min(kKeys, jend - j0);
        __syncthreads();   // the previous block's P, fk, vv are consumed
        kb.store<D + 1, true>(sm.fk, nk, tid);
        vb.store<DV, false>(sm.vv, nk, tid);
        __syncthreads();
        if (j0 + kKeys < jend) {   // the next block's loads fly while this one is used
            kb.load(kf + (size_t)(j0 + kKeys) * D, min(kKeys, jend - j0 - kKeys), tid);
            vb.load(vf + (size_t)(j0 + kKeys) * DV, min(kKeys, jend - j0 - kKeys), tid);
        }
        // P[r][jj] = [j <= i] gamma^(i-j) phi(q_i).phi(k_j), two entries per thread
        for (int e = tid; e < kRows * kKeys; e += kThreads) {
            const int rr = e / kKeys, jj = e % kKeys;
            const int ii = i0 + rr, j = j0 + jj;
            float s = 0.f;
            if (rr < rows && jj < nk && j <= ii) {
#pragma unroll 8
                for (int f = 0; f < D; ++f) s = fmaf(sm.fq[rr][f], sm.fk[jj][f], s);
                s *= expf((float)(ii - j) * lam);
            }
            sm.P[rr][jj] = s;
        }
        __syncthreads();
        for (int jj = 0; jj < nk; ++jj) {
            const float pv = sm.P[r][jj];
            den += pv;
#pragma unroll
            for (int m = 0; m < CPT; ++m) num[m] = fmaf(pv, sm.vv[jj][cl + 16 * m], num[m]);
        }
    }
    if (r >= rows) return;
    // the start state's share
    const float w = expf((float)(i + 1) * lam);
    if (S0) {
        const float* s0 = S0 + chain * (long long)D * DV;
#pragma unroll
        for (int m = 0; m < CPT; ++m) {
            float acc = 0.f;
            for (int f = 0; f < D; ++f) acc = fmaf(sm.fq[r][f], s0[(long long)f * DV + cl + 16 * m], acc);
            num[m] = fmaf(w, acc, num[m]);
        }
    }
    if (z0) {
        const float* zz = z0 + chain * (long long)D;
        float acc = 0.f;
        for (int f = 0; f < D; ++f) acc = fmaf(sm.fq[r][f], zz[f], acc);
        den = fmaf(w, acc, den);
    }
    const float rden = 1.f / (den + eps);
#pragma unroll
    for (int m = 0; m < CPT; ++m) oc[(long long)i * DV + cl + 16 * m] = from_f32<T>(num[m] * rden);
}

// grid (chains, ceil((D*DV + D) / 256)): one state element per thread, the sum
// over the chain's tokens in token order (keys staged through shared memory).
template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads)
kernelized_state_simt(const T* __restrict__ k, const T* __restrict__ v, const float* __restrict__ gamma,
                      const float* __restrict__ S0, const float* __restrict__ z0, float* __restrict__ S_out,
                      float* __restrict__ z_out, int H, int N, int ld)
{
    static_assert(sizeof(T) == 4, "the parallel form stages fp32 rows");
    __shared__ float kt[kKeys][D];
    __shared__ float vt[kKeys][DV];
    __shared__ float wt[kKeys];
    const int tid = threadIdx.x;
    const long long chain = blockIdx.x;
    const int h = (int)(chain % H);
    const float lam = gamma ? logf(gamma[h]) : 0.f;
    const int e = blockIdx.y * kThreads + tid;
    const bool isz = e >= D * DV && e < D * DV + D;
    const bool active = e < D * DV + D;
    const int f = isz ? e - D * DV : e / DV, c = isz ? 0 : e % DV;
    const T* kc = k + chain * (long long)ld * D;
    const T* vc = v + chain * (long long)ld * DV;
    float acc = 0.f;
    const float* kf = reinterpret_cast<const float*>(kc);
    const float* vf = reinterpret_cast<const float*>(vc);
    RowBlock<kKeys, D> kb;
    RowBlock<kKeys, DV> vb;
    kb.load(kf, min(kKeys, N), tid);
    vb.load(vf, min(kKeys, N), tid);
    for (int t0 = 0; t0 < N; t0 += kKeys) {
        const int n = min(kKeys, N - t0);
        __syncthreads();
        kb.store<D, true>(kt, n, tid);
        vb.store<DV, false>(vt, n, tid);
        if (t0 + kKeys < N) {
            kb.load(kf + (size_t)(t0 + kKeys) * D, min(kKeys, N - t0 - kKeys), tid);
            vb.load(vf + (size_t)(t0 + kKeys) * DV, min(kKeys, N - t0 - kKeys), tid);
        }
        if (tid < kKeys) wt[tid] = tid < n ? expf((float)(N - 1 - (t0 + tid)) * lam) : 0.f;
        __syncthreads();
        if (active) {
            if (isz)
                for (int t = 0; t < n; ++t) acc = fmaf(wt[t], kt[t][f], acc);
            else
                for (int t = 0; t < n; ++t) acc = fmaf(wt[t] * kt[t][f], vt[t][c], acc);
        }
    }
    if (!active) return;
    const float wn = expf((float)N * lam);
    if (isz) {
        z_out[chain * D + f] = fmaf(wn, z0 ? z0[chain * D + f] : 0.f, acc);
    } else {
        const long long off = chain * (long long)D * DV + (long long)f * DV + c;
        S_out[off] = fmaf(wn, S0 ? S0[off] : 0.f, acc);
    }
}

template <typename T, int D, int DV>
cudaError_t launch_parallel_t(const PrefillArgs& a)
{
    auto k1 = kernelized_parallel_simt<T, D, DV>;
    const size_t smem = sizeof(ParallelSmem<D, DV>);
    cudaError_t e = cudaFuncSetAttribute(k1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int chains = a.B * a.H;
    k1<<<dim3(chains, (a.N + kRows - 1) / kRows), kThreads, smem, a.stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, a.gamma, a.S0, a.z0, (T*)a.out, a.H, a.N, a.eps, a.ld);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(0, a.stream);
    kernelized_state_simt<T, D, DV><<<dim3(chains, (D * DV + D + kThreads - 1) / kThreads), kThreads, 0, a.stream>>>(
        (const T*)a.k, (const T*)a.v, a.gamma, a.S0, a.z0, a.S_out, a.z_out, a.H, a.N, a.ld);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    stage_mark(1, a.stream);
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_prefill_simt_gla(const PrefillArgs& a)
{
    if (a.dtype == LA_F32) {
        if (a.d == 64) return launch_gla_t<float, 64>(a);
        return launch_gla_t<float, 128>(a);
    }
    if (a.d == 64) return launch_gla_t<__nv_bfloat16, 64>(a);
    return launch_gla_t<__nv_bfloat16, 128>(a);
}

// Sequences of at most kParallelMaxN tokens in fp32 take the parallel form
// (two kernels); longer ones the chunk loop (one kernel).
int simt_kernelized_kernel_count(int N, la_dtype dt) { return dt == LA_F32 && N <= kParallelMaxN ? 2 : 1; }

cudaError_t launch_prefill_simt_kernelized(const PrefillArgs& a)
{
    if (a.dtype == LA_F32) {
        if (a.N <= kParallelMaxN) {
            if (a.d == 64 && a.dv == 64) return launch_parallel_t<float, 64, 64>(a);
            if (a.d == 64 && a.dv == 128) return launch_parallel_t<float, 64, 128>(a);
            if (a.d == 128 && a.dv == 64) return launch_parallel_t<float, 128, 64>(a);
            return launch_parallel_t<float, 128, 128>(a);
        }
        if (a.d == 64) return launch_kernelized_t<float, 64, 32>(a);
        return launch_kernelized_t<float, 128, 32>(a);
    }
    if (a.d == 64) return launch_kernelized_t<__nv_bfloat16, 64, 32>(a);
    return launch_kernelized_t<__nv_bfloat16, 128, 32>(a);
}

cudaError_t launch_prefill_simt_gated_delta(const PrefillArgs& a)
{
    if (a.dtype == LA_F32) {
        if (a.d == 64) return launch_gdelta_t<float, 64>(a);
        return launch_gdelta_t<float, 128>(a);
    }
    if (a.d == 64) return launch_gdelta_t<__nv_bfloat16, 64>(a);
    return launch_gdelta_t<__nv_bfloat16, 128>(a);
}

}  // namespace la
