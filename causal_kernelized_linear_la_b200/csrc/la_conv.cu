// Short causal convolution with a conv cache ("What Is Linear Attention?"
// §5.4: a short convolution over the last w tokens next to the linear state;
// inference keeps a conv cache of the recent tokens' window).
//
// Per chain (b, h) and channel c, with xh = [cache (w-1 rows); x]:
//     y_t[c] = sum_{i=0}^{w-1} W[h][c][i] * xh[t + i][c]      (xh[t + w-1] = x_t)
// and the new cache is the last w-1 rows of xh.
//
// Memory-bound: a thread owns 8 channels (one 16-byte bf16 load, or two
// 16-byte fp32 loads) of a run of kRun consecutive tokens and slides a window
// of the last w-1 rows through registers, so every input row is read once by
// its owner plus w-1 halo rows per run (served by L1/L2); a thread requests
// all of its rows before it uses any.  Arithmetic is fp32 FMA in tap order;
// the output is rounded to the input type once.
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kConvThreads = 256;
constexpr int kRun = 8;   // tokens per thread

// 8 channels of one row in their storage type: one uint4 (bf16) or two float4 (fp32)
template <typename T> struct Raw8;
template <> struct Raw8<__nv_bfloat16> { uint4 a; };
template <> struct Raw8<float> { float4 a, b; };

template <typename T> __device__ __forceinline__ Raw8<T> ldraw(const T* p);
template <> __device__ __forceinline__ Raw8<__nv_bfloat16> ldraw(const __nv_bfloat16* p)
{
    return {*reinterpret_cast<const uint4*>(p)};
}
template <> __device__ __forceinline__ Raw8<float> ldraw(const float* p)
{
    return {reinterpret_cast<const float4*>(p)[0], reinterpret_cast<const float4*>(p)[1]};
}
template <typename T> __device__ __forceinline__ Raw8<T> zraw();
template <> __device__ __forceinline__ Raw8<__nv_bfloat16> zraw() { return {make_uint4(0u, 0u, 0u, 0u)}; }
template <> __device__ __forceinline__ Raw8<float> zraw()
{
    return {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
}
__device__ __forceinline__ void unraw(const Raw8<__nv_bfloat16>& r, float (&f)[8])
{
    const uint32_t w[4] = {r.a.x, r.a.y, r.a.z, r.a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ void unraw(const Raw8<float>& r, float (&f)[8])
{
    f[0] = r.a.x; f[1] = r.a.y; f[2] = r.a.z; f[3] = r.a.w;
    f[4] = r.b.x; f[5] = r.b.y; f[6] = r.b.z; f[7] = r.b.w;
}

template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&f)[8]);
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16* p, float (&f)[8])
{
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
template <>
__device__ __forceinline__ void load8<float>(const float* p, float (&f)[8])
{
    const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&f)[8]);
template <>
__device__ __forceinline__ void store8<__nv_bfloat16>(__nv_bfloat16* p, const float (&f)[8])
{
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
template <>
__device__ __forceinline__ void store8<float>(float* p, const float (&f)[8])
{
    reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

// grid: (token tiles, chains); block: kConvThreads threads = (d / 8) channel
// groups x lanes token lanes, each lane kRun tokens.
template <typename T, int W>
__global__ void __launch_bounds__(kConvThreads)
causal_conv_kernel(const T* __restrict__ x, const float* __restrict__ weight, const T* __restrict__ cache,
                   T* __restrict__ y, T* __restrict__ cache_out, int H, int N, int d)
{
    constexpr int HIST = W - 1;
    const int groups = d / 8;
    const int lanes = kConvThreads / groups;
    const int cg = threadIdx.x % groups, lane = threadIdx.x / groups;
    const int chain = blockIdx.y, h = chain % H;
    const int c0 = cg * 8;
    const T* xc = x + (size_t)chain * N * d + c0;
    const T* cc = cache ? cache + (size_t)chain * HIST * d + c0 : nullptr;

    // row r of [cache; x] (r may be < HIST: the history), 8 channels
    auto row = [&](int r, float (&f)[8]) {
        if (r >= HIST) {
            load8<T>(xc + (size_t)(r - HIST) * d, f);
        } else if (cc) {
            load8<T>(cc + (size_t)r * d, f);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) f[j] = 0.f;
        }
    };

    // the new cache: the first block of every chain writes rows 0..W-2
    if (cache_out && blockIdx.x == 0) {
        for (int r = lane; r < HIST; r += lanes) {
            float f[8];
            row(N + r, f);
            store8<T>(cache_out + ((size_t)chain * HIST + r) * d + c0, f);
        }
    }

    const int t0 = (blockIdx.x * lanes + lane) * kRun;
    if (t0 >= N) return;
    const int t1 = min(N, t0 + kRun);

    // every row this thread needs is requested before any is used, so the
    // loads overlap instead of costing one memory latency per token
    Raw8<T> raw[kRun + HIST];
#pragma unroll
    for (int r = 0; r < kRun + HIST; ++r) {
        const int k = t0 + r;                      // row of [cache; x]
        if (k >= HIST) raw[r] = (k - HIST < N) ? ldraw<T>(xc + (size_t)(k - HIST) * d) : zraw<T>();
        else raw[r] = cc ? ldraw<T>(cc + (size_t)k * d) : zraw<T>();
    }
    float wt[W][8];
    {
        const float* wp = weight + ((size_t)h * d + c0) * W;   // [8 channels][W taps], contiguous
#pragma unroll
        for (int j = 0; j < 8; ++j)
#pragma unroll
            for (int i = 0; i < W; ++i) wt[i][j] = wp[j * W + i];
    }
    // window: win[i] = xh[t + i] for the next output t
    float win[W][8];
#pragma unroll
    for (int i = 0; i < HIST; ++i) unraw(raw[i], win[i]);
    T* yc = y + (size_t)chain * N * d + c0;
#pragma unroll
    for (int u = 0; u < kRun; ++u) {
        unraw(raw[u + HIST], win[HIST]);
        float acc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
        for (int i = 0; i < W; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[j] = fmaf(wt[i][j], win[i][j], acc[j]);
        if (t0 + u < t1) store8<T>(yc + (size_t)(t0 + u) * d, acc);
#pragma unroll
        for (int i = 0; i < HIST; ++i)
#pragma unroll
            for (int j = 0; j < 8; ++j) win[i][j] = win[i + 1][j];
    }
}

template <typename T, int W>
cudaError_t launch_conv_t(const ConvArgs& a)
{
    const int groups = a.d / 8, lanes = kConvThreads / groups;
    const int tile = lanes * kRun;
    const int tiles = a.N > 0 ? (a.N + tile - 1) / tile : 1;
    dim3 grid(tiles, a.B * a.H);
    causal_conv_kernel<T, W><<<grid, kConvThreads, 0, a.stream>>>(
        (const T*)a.x, a.weight, (const T*)a.cache, (T*)a.y, (T*)a.cache_out, a.H, a.N, a.d);
    const cudaError_t e = cudaGetLastError();
    if (e == cudaSuccess) stage_mark(0, a.stream);
    return e;
}

template <typename T>
cudaError_t launch_conv_dt(const ConvArgs& a)
{
    switch (a.w) {
        case 1: return launch_conv_t<T, 1>(a);
        case 2: return launch_conv_t<T, 2>(a);
        case 3: return launch_conv_t<T, 3>(a);
        case 4: return launch_conv_t<T, 4>(a);
        case 5: return launch_conv_t<T, 5>(a);
        case 6: return launch_conv_t<T, 6>(a);
        case 7: return launch_conv_t<T, 7>(a);
        case 8: return launch_conv_t<T, 8>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_causal_conv(const ConvArgs& a)
{
    return a.dtype == LA_BF16 ? launch_conv_dt<__nv_bfloat16>(a) : launch_conv_dt<float>(a);
}

}  // namespace la
