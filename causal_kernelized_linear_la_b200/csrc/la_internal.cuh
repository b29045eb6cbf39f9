// Internal declarations shared by the library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "la.h"

namespace la {

// Everything one prefill launch needs, already validated by the API layer.
struct PrefillArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* gamma;  // [H] (LA_DECAY) or nullptr
    const float* alpha;  // [B,H,N] (LA_GATED_DELTA) or nullptr
    const float* g;      // [B,H,N] (LA_GATED_DELTA) or nullptr
    void* out;
    float* S_out;
    float* z_out;
    const float* S0;
    const float* z0;
    int B, H, N, d, dv;
    // tokens between the first rows of consecutive (b, h) chains of q, k, v,
    // out, alpha and g: N for a dense [B,H,N,.] batch, the padded length when
    // one sequence of a right-padded batch is run over its own length
    int ld;
    // launch the call's first kernel with programmatic serialization: it may
    // start while the stream's previous kernels drain (it reads none of their
    // results and finishes after them); only for back-to-back calls of one
    // batch whose workspaces are disjoint
    bool pdl_first;
    float eps;
    la_dtype dtype;
    la_mode mode;
    cudaStream_t stream;
    void* workspace;
    size_t workspace_bytes;
};

struct DecodeArgs {
    const void* q;
    const void* k;
    const void* v;
    const float* alpha;  // gated delta only
    const float* g;      // gated delta only
    float* S;
    float* z;            // kernelized only
    void* out;
    int B, H, d, dv;
    float eps;
    la_dtype dtype;
    cudaStream_t stream;
};

struct ConvArgs {
    const void* x;
    const float* weight;
    const void* cache;   // may be null: zero history
    void* y;
    void* cache_out;     // may be null
    int B, H, N, d, w;
    la_dtype dtype;
    cudaStream_t stream;
};

bool uses_tc_kernelized(la_dtype dt, la_mode m);

// Short causal convolution with conv cache (memory-bound SIMT).
cudaError_t launch_causal_conv(const ConvArgs& a);

// SIMT prefill kernels (fp32 arithmetic; fp32 or bf16 inputs).
cudaError_t launch_prefill_simt_kernelized(const PrefillArgs& a);
// kernels one fp32 kernelized prefill of N tokens launches (the parallel form for short sequences)
int simt_kernelized_kernel_count(int N, la_dtype dt);
cudaError_t launch_prefill_simt_gated_delta(const PrefillArgs& a);
cudaError_t launch_prefill_simt_gla(const PrefillArgs& a);

// Decode kernels (HBM-streaming SIMT).
cudaError_t launch_decode_kernelized(const DecodeArgs& a);
cudaError_t launch_decode_gated_delta(const DecodeArgs& a);

// ---------------------------------------------------------------------------
// Small device helpers used by several kernels.

// elu(x) + 1 with alpha = 1: x + 1 for x > 0, exp(x) otherwise
// ("Efficient attention variants" §4).  Only the non-positive branch calls
// exp, so no large exponent is ever evaluated.  phi() uses the accurate expf
// (fp32-input paths); phi_fast() the SFU __expf, whose error is far below the
// bf16 rounding applied right after it on the tensor-core paths.
__device__ __forceinline__ float phi(float x) { return x > 0.f ? x + 1.f : expf(x); }
__device__ __forceinline__ float phi_fast(float x) { return x > 0.f ? x + 1.f : __expf(x); }

template <typename T> __device__ __forceinline__ float to_f32(T x);
template <> __device__ __forceinline__ float to_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// Profiling hook (la_set_stage_events): record the caller's i-th event on
// `stream` right after a call's i-th kernel launch, if one is set.
void stage_mark(int i, cudaStream_t stream);

// Failure-path self-test of the bounded waits (la_selftest.cu): one kernel
// whose mbarrier wait runs out, and the reader of that unit's error word.
cudaError_t launch_wait_timeout_selftest(cudaStream_t stream);
unsigned int read_and_clear_device_error_selftest(cudaStream_t stream);

}  // namespace la
