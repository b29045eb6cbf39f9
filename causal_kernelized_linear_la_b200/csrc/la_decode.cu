// Decode-step kernels: one token per (sequence, head) against a resident fp32
// state.  The state is the whole cache ("What Is Linear Attention?" §6), so a
// step reads and writes d*dv*4 bytes per (sequence, head) and does ~4 flops
// per element: the step is bound by HBM bandwidth and nothing else.
//
// Layout of one block's work: the state S [d][dv] of one (sequence, head) is
// streamed exactly once.  A thread owns 4 adjacent columns (one 16-byte
// vector) of d / (rows per block step) rows; its loads are all issued before
// any arithmetic so that a block keeps its whole 32-64 KB tile in flight.
// Loads and stores use the streaming cache hint: the state is far larger than
// L2 and is not re-read within a step.
//
// kernelized ("What Is Linear Attention?" §4, order: write then read):
//   S[i,:] += phi(k_i) v;  num = sum_i phi(q_i) S[i,:];  z += phi(k);
//   den = phi(q).z;  out = num / (den + eps)
// gated delta ("Efficient attention variants" §7.4):
//   vhat = S^T k;  S = alpha S + g k (v - alpha vhat)^T;  out = S^T q
// The delta step needs S^T k before the write; the tile stays in registers
// between the two reductions so S is still read and written once.
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

template <int D, int DV>
struct DecodeGeom {
    static constexpr int LPR = DV / 4;                 // lanes per state row
    static constexpr int RPW = 32 / LPR;               // rows per warp per step
    static constexpr int RG = kWarps * RPW;            // row groups per block
    static constexpr int RPT = D / RG;                 // rows per thread
    static_assert(D % RG == 0, "rows must divide evenly");
};

template <typename T> __device__ __forceinline__ float ld_in(const T* p) { return to_f32(*p); }

// Sum float4 partials of all row groups; result for column c in red_out[c].
template <int DV, int RG>
__device__ __forceinline__ void reduce_columns(float (*red)[DV], const float4& acc, int rg, int c4,
                                               float* red_out)
{
    *reinterpret_cast<float4*>(&red[rg][c4 * 4]) = acc;
    __syncthreads();
    for (int c = threadIdx.x; c < DV; c += kThreads) {
        float s = 0.f;
#pragma unroll
        for (int r = 0; r < RG; ++r) s += red[r][c];
        red_out[c] = s;
    }
    __syncthreads();
}

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads)
decode_kernelized(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  float* __restrict__ S, float* __restrict__ z, T* __restrict__ out, float eps)
{
    using G = DecodeGeom<D, DV>;
    __shared__ __align__(16) float fq[D];
    __shared__ __align__(16) float fk[D];
    __shared__ __align__(16) float vs[DV];
    __shared__ __align__(16) float red[G::RG][DV];
    __shared__ float num[DV];
    __shared__ float den_part[kWarps];

    const long long st = blockIdx.x;  // (sequence, head) index
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c4 = lane % G::LPR;
    const int rg = warp * G::RPW + lane / G::LPR;
    float4* Sp = reinterpret_cast<float4*>(S + st * (long long)D * DV);

    // 1. the whole state tile goes in flight first
    float4 s[G::RPT];
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) s[r] = __ldcs(Sp + (long long)(rg + r * G::RG) * G::LPR + c4);

    // 2. the token: features, value, normaliser (while the loads are in flight)
    float dpart = 0.f;
    for (int i = threadIdx.x; i < D; i += kThreads) {
        const float a = phi(ld_in(q + st * D + i));
        const float b = phi(ld_in(k + st * D + i));
        fq[i] = a;
        fk[i] = b;
        const float zi = z[st * D + i] + b;   // z_t = z_{t-1} + phi(k_t)
        z[st * D + i] = zi;
        dpart = fmaf(a, zi, dpart);
    }
    for (int j = threadIdx.x; j < DV; j += kThreads) vs[j] = ld_in(v + st * DV + j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    if (lane == 0) den_part[warp] = dpart;
    __syncthreads();

    // 3. fused write + read over the tile: S += phi(k) v^T; acc += phi(q) S
    const float4 v4 = *reinterpret_cast<const float4*>(&vs[c4 * 4]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
        const int row = rg + r * G::RG;
        const float b = fk[row], a = fq[row];
        float4 x = s[r];
        x.x = fmaf(b, v4.x, x.x);
        x.y = fmaf(b, v4.y, x.y);
        x.z = fmaf(b, v4.z, x.z);
        x.w = fmaf(b, v4.w, x.w);
        __stcs(Sp + (long long)row * G::LPR + c4, x);
        acc.x = fmaf(a, x.x, acc.x);
        acc.y = fmaf(a, x.y, acc.y);
        acc.z = fmaf(a, x.z, acc.z);
        acc.w = fmaf(a, x.w, acc.w);
    }
    reduce_columns<DV, G::RG>(red, acc, rg, c4, num);

    float den = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) den += den_part[w];
    const float inv = 1.f / (den + eps);
    for (int j = threadIdx.x; j < DV; j += kThreads) out[st * DV + j] = from_f32<T>(num[j] * inv);
}

template <typename T, int D, int DV>
__global__ void __launch_bounds__(kThreads)
decode_gated_delta(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ alpha, const float* __restrict__ g,
                   float* __restrict__ S, T* __restrict__ out)
{
    using G = DecodeGeom<D, DV>;
    __shared__ __align__(16) float qs[D];
    __shared__ __align__(16) float ks[D];
    __shared__ __align__(16) float vs[DV];
    __shared__ __align__(16) float red[G::RG][DV];
    __shared__ __align__(16) float vhat[DV];
    __shared__ float ob[DV];

    const long long st = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c4 = lane % G::LPR;
    const int rg = warp * G::RPW + lane / G::LPR;
    float4* Sp = reinterpret_cast<float4*>(S + st * (long long)D * DV);

    float4 s[G::RPT];
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) s[r] = __ldcs(Sp + (long long)(rg + r * G::RG) * G::LPR + c4);

    for (int i = threadIdx.x; i < D; i += kThreads) {
        qs[i] = ld_in(q + st * D + i);
        ks[i] = ld_in(k + st * D + i);
    }
    for (int j = threadIdx.x; j < DV; j += kThreads) vs[j] = ld_in(v + st * DV + j);
    const float a = alpha[st], gg = g[st];
    __syncthreads();

    // vhat = S_{t-1}^T k
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
        const float kr = ks[rg + r * G::RG];
        acc.x = fmaf(kr, s[r].x, acc.x);
        acc.y = fmaf(kr, s[r].y, acc.y);
        acc.z = fmaf(kr, s[r].z, acc.z);
        acc.w = fmaf(kr, s[r].w, acc.w);
    }
    reduce_columns<DV, G::RG>(red, acc, rg, c4, vhat);

    // err = g (v - alpha vhat);  S = alpha S + k err^T;  o = S^T q
    const float4 v4 = *reinterpret_cast<const float4*>(&vs[c4 * 4]);
    const float4 h4 = *reinterpret_cast<const float4*>(&vhat[c4 * 4]);
    const float4 e4 = make_float4(gg * (v4.x - a * h4.x), gg * (v4.y - a * h4.y),
                                  gg * (v4.z - a * h4.z), gg * (v4.w - a * h4.w));
    acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < G::RPT; ++r) {
        const int row = rg + r * G::RG;
        const float kr = ks[row], qr = qs[row];
        float4 x = s[r];
        x.x = fmaf(a, x.x, kr * e4.x);
        x.y = fmaf(a, x.y, kr * e4.y);
        x.z = fmaf(a, x.z, kr * e4.z);
        x.w = fmaf(a, x.w, kr * e4.w);
        __stcs(Sp + (long long)row * G::LPR + c4, x);
        acc.x = fmaf(qr, x.x, acc.x);
        acc.y = fmaf(qr, x.y, acc.y);
        acc.z = fmaf(qr, x.z, acc.z);
        acc.w = fmaf(qr, x.w, acc.w);
    }
    reduce_columns<DV, G::RG>(red, acc, rg, c4, ob);
    for (int j = threadIdx.x; j < DV; j += kThreads) out[st * DV + j] = from_f32<T>(ob[j]);
}

template <typename T, int D, int DV>
cudaError_t launch_kz(const DecodeArgs& a)
{
    const long long n = (long long)a.B * a.H;
    decode_kernelized<T, D, DV><<<(unsigned)n, kThreads, 0, a.stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, a.S, a.z, (T*)a.out, a.eps);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) stage_mark(0, a.stream);
    return e;
}

template <typename T, int D, int DV>
cudaError_t launch_gd(const DecodeArgs& a)
{
    const long long n = (long long)a.B * a.H;
    decode_gated_delta<T, D, DV><<<(unsigned)n, kThreads, 0, a.stream>>>(
        (const T*)a.q, (const T*)a.k, (const T*)a.v, a.alpha, a.g, a.S, (T*)a.out);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) stage_mark(0, a.stream);
    return e;
}

}  // namespace

#define LA_DECODE_DISPATCH(FN, a)                                                      \
    do {                                                                               \
        if ((a).dtype == LA_F32) {                                                     \
            if ((a).d == 64 && (a).dv == 64) return FN<float, 64, 64>(a);              \
            if ((a).d == 64 && (a).dv == 128) return FN<float, 64, 128>(a);            \
            if ((a).d == 128 && (a).dv == 64) return FN<float, 128, 64>(a);            \
            return FN<float, 128, 128>(a);                                             \
        }                                                                              \
        if ((a).d == 64 && (a).dv == 64) return FN<__nv_bfloat16, 64, 64>(a);          \
        if ((a).d == 64 && (a).dv == 128) return FN<__nv_bfloat16, 64, 128>(a);        \
        if ((a).d == 128 && (a).dv == 64) return FN<__nv_bfloat16, 128, 64>(a);        \
        return FN<__nv_bfloat16, 128, 128>(a);                                         \
    } while (0)

cudaError_t launch_decode_kernelized(const DecodeArgs& a) { LA_DECODE_DISPATCH(launch_kz, a); }
cudaError_t launch_decode_gated_delta(const DecodeArgs& a) { LA_DECODE_DISPATCH(launch_gd, a); }

}  // namespace la
