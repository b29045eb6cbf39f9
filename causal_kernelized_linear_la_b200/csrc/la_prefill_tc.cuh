// Host-side interface of the tensor-core prefill kernels.
#pragma once

#include <cuda.h>

#include "la_internal.cuh"

namespace la {

// Sequence split of the tensor-core prefill: segments of L tokens (a multiple
// of the 64-token chunk), G segments per (batch, head) chain.
struct TcSegments {
    int L = 0;
    int G = 0;
};

TcSegments tc_segments(int B, int H, int N, int d, int dv);

// Segment map of one launch set of the kernelized tensor-core prefill: either a
// uniform batch (every chain has N tokens in G segments of L) or a right-padded
// batch of up to kMaxVarlenSeqs sequences of their own lengths (sequence b: H
// chains of lens[b] tokens in ceil(lens[b] / L) segments; units are numbered
// sequence by sequence, head by head, segment by segment).
constexpr int kMaxVarlenSeqs = 64;
struct SegMap {
    int H = 0;
    int L = 0;
    int B = 0;   // 0: uniform batch
    int N = 0;   // uniform: tokens per chain
    int G = 0;   // uniform: segments per chain
    int lens[kMaxVarlenSeqs] = {};
};
size_t tc_workspace_bytes(int B, int H, int N, int d, int dv);
cudaError_t launch_prefill_tc_kernelized(const PrefillArgs& a);

// One launch set over a right-padded batch (a.B <= kMaxVarlenSeqs sequences,
// a.N = a.ld = the padded length): segment length and workspace slots.
int varlen_segment_length(const int* lens, int B, int H, int d, int dv);
size_t tc_varlen_workspace_bytes(const int* lens, int B, int H, int d, int dv);
cudaError_t launch_prefill_tc_kernelized_varlen(const PrefillArgs& a, const int* lens);

// Fixed scratch of the no-allocation entry point (la_prefill_noalloc).
constexpr size_t kNoAllocScratchBytes = 16u << 20;
TcSegments tc_segments_noalloc(int B, int H, int N, int d, int dv);
cudaError_t launch_prefill_tc_kernelized_noalloc(const PrefillArgs& a);
// Device address of that scratch on the current device (looked up once per device).
void* noalloc_scratch_address(cudaError_t* err);

// GLA (per-key-channel gate) on the tensor cores, bf16 inputs: segment
// summaries, scan, chunk loop; the workspace (or the fixed scratch) holds one
// d x dv + d slot per (chain, segment), as for the kernelized modes.
cudaError_t launch_prefill_tc_gla(const PrefillArgs& a, const TcSegments& sg);
unsigned int read_and_clear_device_error_gla(cudaStream_t stream);

// 3-D TMA map over the first N rows of each chain of a bf16 tensor whose
// chains start ld rows apart ([chains][ld][inner], ld >= N); box 64 x 64
// rows, 128-byte swizzle, zero fill past N, stores clipped at N.
bool make_map(CUtensorMap* m, const void* base, int inner, int N, int chains, int ld);

// Gated-delta prefill on the tensor cores (bf16 inputs).  The workspace holds
// the per-chunk operands the parallel pass hands to the sequential pass.  A
// long sequence runs as up to kMaxGdParts parts (whole 64-token chunks, the
// last part excepted; each part longer than the one before) whose passes
// overlap; a call launches 2 P kernels.
constexpr int kMaxGdParts = 8;
struct GdParts {
    int P = 1;
    int start[kMaxGdParts + 1] = {};   // part i is tokens start[i] .. start[i + 1] - 1
};
GdParts gd_parts(int B, int H, int N, int d, int dv);
size_t gd_workspace_bytes(int B, int H, int N, int d, int dv);
cudaError_t launch_prefill_tc_gated_delta(const PrefillArgs& a);
unsigned int read_and_clear_device_error_gdelta(cudaStream_t stream);

// Read (and clear) the device error word the tensor-core kernels set when a
// bounded wait gives up.  Synchronises `stream`.
unsigned int read_and_clear_device_error(cudaStream_t stream);

}  // namespace la
