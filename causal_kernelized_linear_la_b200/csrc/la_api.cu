// C ABI entry points: argument validation and dispatch to the kernels.
// Nothing here computes; every step of the path runs in the kernels.
#include <stdint.h>

#include "la_internal.cuh"
#include "la_prefill_tc.cuh"

namespace la {
namespace {

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool head_ok(int x) { return x == 64 || x == 128; }

// Byte ranges [a, a + na) and [b, b + nb) share at least one byte.
bool overlap(const void* a, size_t na, const void* b, size_t nb)
{
    if (!a || !b || na == 0 || nb == 0) return false;
    const char* pa = static_cast<const char*>(a);
    const char* pb = static_cast<const char*>(b);
    return pa < pb + nb && pb < pa + na;
}

// The final-state outputs of a prefill share no byte with its start state:
// blocks of one call read S0 / z0 while others write S_out / z_out.
bool state_outputs_alias(const float* S_out, const float* z_out, const float* S0, const float* z0, int B, int H, int d,
                         int dv)
{
    const size_t chains = (size_t)B * H;
    const size_t sb = chains * d * dv * sizeof(float), zb = chains * d * sizeof(float);
    const void* outs[2] = {S_out, z_out};
    const size_t on[2] = {sb, zb};
    const void* ins[2] = {S0, z0};
    const size_t in_n[2] = {sb, zb};
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 2; ++j)
            if (overlap(outs[i], on[i], ins[j], in_n[j])) return true;
    return false;
}

// Stage events of la_set_stage_events (process-wide; see la.h).
constexpr int kMaxStageEvents = 16;
cudaEvent_t g_stage_events[kMaxStageEvents];
int g_stage_count = 0;

la_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LA_OK : LA_ERR_CUDA; }

}  // namespace

void stage_mark(int i, cudaStream_t stream)
{
    if (i < g_stage_count) cudaEventRecord(g_stage_events[i], stream);
}

// bf16 kernelized prefill runs on the tensor cores; fp32 inputs stay on the
// fp32 SIMT kernels (bf16 operands could not meet a 1e-4 error bound).
bool uses_tc_kernelized(la_dtype dt, la_mode m) { return dt == LA_BF16 && (m == LA_PLAIN || m == LA_DECAY); }

namespace {

// Final state for an empty sequence: the start state, or zero.
la_status write_start_state(const PrefillArgs& a)
{
    const size_t chains = (size_t)a.B * a.H;
    const size_t sbytes = chains * a.d * a.dv * sizeof(float);
    const size_t zbytes = chains * a.d * sizeof(float);
    cudaError_t e = cudaSuccess;
    if (a.S0) e = cudaMemcpyAsync(a.S_out, a.S0, sbytes, cudaMemcpyDeviceToDevice, a.stream);
    else e = cudaMemsetAsync(a.S_out, 0, sbytes, a.stream);
    if (e == cudaSuccess && a.z_out) {
        if (a.z0) e = cudaMemcpyAsync(a.z_out, a.z0, zbytes, cudaMemcpyDeviceToDevice, a.stream);
        else e = cudaMemsetAsync(a.z_out, 0, zbytes, a.stream);
    }
    return from_cuda(e);
}

// Argument checks of a prefill over a [B,H,N,.] batch (all but the workspace size).
la_status check_prefill(const void* q, const void* k, const void* v, const float* gamma_or_alpha, const float* g,
                        const void* out, const float* S_out, const float* z_out, int B, int H, int N, int d, int dv,
                        const la_config* cfg)
{
    if (!cfg) return LA_ERR_INVALID;
    if (B < 0 || H < 0 || N < 0) return LA_ERR_INVALID;
    if (cfg->dtype != LA_F32 && cfg->dtype != LA_BF16) return LA_ERR_INVALID;
    if (cfg->mode != LA_PLAIN && cfg->mode != LA_DECAY && cfg->mode != LA_GATED_DELTA && cfg->mode != LA_GLA)
        return LA_ERR_INVALID;
    if (!head_ok(d) || !head_ok(dv)) return LA_ERR_UNSUPPORTED;
    const bool delta = cfg->mode == LA_GATED_DELTA;
    const bool gla = cfg->mode == LA_GLA;
    const bool no_norm = delta || gla;   // modes without the z normaliser
    const bool work = (long long)B * H > 0;
    if (work) {
        if (!S_out) return LA_ERR_INVALID;
        if (!no_norm && !z_out) return LA_ERR_INVALID;
        if (no_norm && z_out) return LA_ERR_INVALID;
        if (N > 0 && (!q || !k || !v || !out)) return LA_ERR_INVALID;
        if (cfg->mode == LA_PLAIN && (gamma_or_alpha || g)) return LA_ERR_INVALID;
        if (cfg->mode == LA_DECAY && (!gamma_or_alpha || g)) return LA_ERR_INVALID;
        if (delta && N > 0 && (!gamma_or_alpha || !g)) return LA_ERR_INVALID;
        if (gla && (g || (N > 0 && !gamma_or_alpha))) return LA_ERR_INVALID;
    }
    if (!(cfg->eps >= 0.f)) return LA_ERR_INVALID;
    if (work && state_outputs_alias(S_out, z_out, cfg->S0, no_norm ? nullptr : cfg->z0, B, H, d, dv))
        return LA_ERR_INVALID;
    const void* ptrs[] = {q, k, v, gamma_or_alpha, g, out, S_out, z_out, cfg->S0, cfg->z0, cfg->workspace};
    for (const void* p : ptrs)
        if (!aligned16(p)) return LA_ERR_ALIGN;
    return LA_OK;
}

PrefillArgs prefill_args(const void* q, const void* k, const void* v, const float* gamma_or_alpha, const float* g,
                         void* out, float* S_out, float* z_out, int B, int H, int N, int d, int dv,
                         const la_config* cfg)
{
    const bool delta = cfg->mode == LA_GATED_DELTA;
    const bool no_norm = delta || cfg->mode == LA_GLA;
    PrefillArgs a{};
    a.q = q; a.k = k; a.v = v;
    a.gamma = cfg->mode == LA_DECAY ? gamma_or_alpha : nullptr;
    a.alpha = no_norm ? gamma_or_alpha : nullptr;
    a.g = delta ? g : nullptr;
    a.out = out; a.S_out = S_out; a.z_out = no_norm ? nullptr : z_out;
    a.S0 = cfg->S0; a.z0 = no_norm ? nullptr : cfg->z0;
    a.B = B; a.H = H; a.N = N; a.d = d; a.dv = dv;
    a.ld = N;
    a.eps = cfg->eps; a.dtype = cfg->dtype; a.mode = cfg->mode;
    a.stream = static_cast<cudaStream_t>(cfg->stream);
    a.workspace = cfg->workspace; a.workspace_bytes = cfg->workspace_bytes;
    return a;
}

// A right-padded batch runs as one launch set (instead of one per sequence)
// on the bf16 tensor-core path of the kernelized modes, up to kMaxVarlenSeqs
// sequences.
bool varlen_one_launch_set(const int* lens, int B, int H, int d, int dv, const la_config* cfg)
{
    if (!cfg || !lens || B <= 0 || B > kMaxVarlenSeqs || H <= 0 || !head_ok(d) || !head_ok(dv)) return false;
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0) return false;
    return uses_tc_kernelized(cfg->dtype, cfg->mode);
}

// Workspace slice of one sequence of la_prefill_varlen: 256-byte aligned.
size_t varlen_slice(size_t bytes) { return (bytes + 255) / 256 * 256; }

// One checked prefill to the kernels of its dtype and mode.
la_status run_prefill(const PrefillArgs& a)
{
    if (a.N == 0) return write_start_state(a);
    if (a.mode == LA_GLA) {
        if (a.dtype == LA_BF16) return from_cuda(launch_prefill_tc_gla(a, tc_segments(a.B, a.H, a.N, a.d, a.dv)));
        return from_cuda(launch_prefill_simt_gla(a));
    }
    if (a.mode == LA_GATED_DELTA) {
        if (a.dtype == LA_BF16) return from_cuda(launch_prefill_tc_gated_delta(a));
        return from_cuda(launch_prefill_simt_gated_delta(a));
    }
    if (uses_tc_kernelized(a.dtype, a.mode)) return from_cuda(launch_prefill_tc_kernelized(a));
    return from_cuda(launch_prefill_simt_kernelized(a));
}

}  // namespace
}  // namespace la

using la::PrefillArgs;
using la::DecodeArgs;

extern "C" {

const char* la_version(void) { return "0.1.0"; }

const char* la_status_string(la_status s)
{
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID: return "LA_ERR_INVALID: invalid argument";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: head size or dtype/mode not supported";
        case LA_ERR_ALIGN: return "LA_ERR_ALIGN: pointer not 16-byte aligned";
        case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA call or kernel launch failed";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT: a bounded device-side wait gave up";
        case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    }
    return "unknown la_status";
}

size_t la_prefill_workspace_bytes(int B, int H, int N, int d, int dv, const la_config* cfg)
{
    if (!cfg || B <= 0 || H <= 0 || N <= 0 || !la::head_ok(d) || !la::head_ok(dv)) return 0;
    if (la::uses_tc_kernelized(cfg->dtype, cfg->mode)) return la::tc_workspace_bytes(B, H, N, d, dv);
    if (cfg->dtype == LA_BF16 && cfg->mode == LA_GLA) return la::tc_workspace_bytes(B, H, N, d, dv);
    if (cfg->dtype == LA_BF16 && cfg->mode == LA_GATED_DELTA) return la::gd_workspace_bytes(B, H, N, d, dv);
    return 0;
}

int la_prefill_kernel_count(int B, int H, int N, int d, int dv, const la_config* cfg)
{
    if (!cfg || B <= 0 || H <= 0 || N <= 0 || !la::head_ok(d) || !la::head_ok(dv)) return 0;
    if (la::uses_tc_kernelized(cfg->dtype, cfg->mode)) return 3;
    if (cfg->dtype == LA_BF16 && cfg->mode == LA_GLA) return 3;
    if (cfg->dtype == LA_BF16 && cfg->mode == LA_GATED_DELTA) return 2 * la::gd_parts(B, H, N, d, dv).P;
    if (cfg->mode == LA_PLAIN || cfg->mode == LA_DECAY) return la::simt_kernelized_kernel_count(N, cfg->dtype);
    return 1;
}

la_status la_prefill(const void* q, const void* k, const void* v,
                     const float* gamma_or_alpha, const float* g,
                     void* out, float* S_out, float* z_out,
                     int B, int H, int N, int d, int dv, const la_config* cfg)
{
    const la_status st = la::check_prefill(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, cfg);
    if (st != LA_OK) return st;
    if (cfg->workspace_bytes < la_prefill_workspace_bytes(B, H, N, d, dv, cfg)) return LA_ERR_WORKSPACE;
    if ((long long)B * H == 0) return LA_OK;
    return la::run_prefill(la::prefill_args(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, cfg));
}

size_t la_prefill_varlen_workspace_bytes(const int* seq_lens, int B, int H, int d, int dv, const la_config* cfg)
{
    if (!seq_lens || B <= 0) return 0;
    if (la::varlen_one_launch_set(seq_lens, B, H, d, dv, cfg))
        return la::tc_varlen_workspace_bytes(seq_lens, B, H, d, dv);
    size_t total = 0;
    for (int b = 0; b < B; ++b) total += la::varlen_slice(la_prefill_workspace_bytes(1, H, seq_lens[b], d, dv, cfg));
    return total;
}

la_status la_prefill_varlen(const void* q, const void* k, const void* v,
                            const float* gamma_or_alpha, const float* g,
                            void* out, float* S_out, float* z_out, const int* seq_lens,
                            int B, int H, int N, int d, int dv, const la_config* cfg)
{
    const la_status st = la::check_prefill(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, cfg);
    if (st != LA_OK) return st;
    if ((long long)B * H == 0) return LA_OK;
    if (!seq_lens) return LA_ERR_INVALID;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] < 0 || seq_lens[b] > N) return LA_ERR_INVALID;
    if (cfg->workspace_bytes < la_prefill_varlen_workspace_bytes(seq_lens, B, H, d, dv, cfg))
        return LA_ERR_WORKSPACE;

    // Sequence b is the B = 1 batch of its H chains over its own length; its
    // chains keep the batch's row stride N, so the padding rows are neither
    // read (the TMA maps and the SIMT loops end at the length) nor written.
    // Each sequence has a slice of the workspace of its own, so the first
    // kernel of sequence b > 0 may start while sequence b-1's kernels drain
    // (programmatic serialization); it finishes after them.
    const PrefillArgs base = la::prefill_args(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, cfg);
    if (la::varlen_one_launch_set(seq_lens, B, H, d, dv, cfg)) {
        // one launch set over every sequence of the batch
        bool any = false;
        for (int b = 0; b < B; ++b) any = any || seq_lens[b] > 0;
        if (!any) return la::write_start_state(base);
        return la::from_cuda(la::launch_prefill_tc_kernelized_varlen(base, seq_lens));
    }
    const size_t esz = cfg->dtype == LA_BF16 ? 2 : 4;
    size_t ws_off = 0;
    for (int b = 0; b < B; ++b) {
        PrefillArgs a = base;
        const size_t ws_b = la_prefill_workspace_bytes(1, H, seq_lens[b], d, dv, cfg);
        a.workspace = ws_b ? static_cast<char*>(cfg->workspace) + ws_off : nullptr;
        a.workspace_bytes = ws_b;
        ws_off += la::varlen_slice(ws_b);
        a.pdl_first = b > 0 && seq_lens[b - 1] > 0;   // behind a kernel of sequence b-1
        const size_t row0 = (size_t)b * H * N;   // first row of sequence b
        const size_t st_s = (size_t)b * H * d * dv, st_z = (size_t)b * H * d;
        a.q = static_cast<const char*>(q) + row0 * d * esz;
        a.k = static_cast<const char*>(k) + row0 * d * esz;
        a.v = static_cast<const char*>(v) + row0 * dv * esz;
        a.out = static_cast<char*>(out) + row0 * dv * esz;
        if (a.alpha) a.alpha += cfg->mode == LA_GLA ? row0 * d : row0;
        if (a.g) a.g += row0;
        a.S_out += st_s;
        if (a.z_out) a.z_out += st_z;
        if (a.S0) a.S0 += st_s;
        if (a.z0) a.z0 += st_z;
        a.B = 1;
        a.N = seq_lens[b];
        a.ld = N;
        const la_status r = la::run_prefill(a);
        if (r != LA_OK) return r;
    }
    return LA_OK;
}

la_status la_prefill_noalloc(const void* q, const void* k, const void* v,
                             const float* gamma_or_alpha, const float* g,
                             void* out, float* S_out, float* z_out,
                             int B, int H, int N, int d, int dv, const la_config* cfg)
{
    if (!cfg) return LA_ERR_INVALID;
    la_config c = *cfg;   // cfg->workspace is ignored
    c.workspace = nullptr;
    c.workspace_bytes = 0;
    const la_status st = la::check_prefill(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, &c);
    if (st != LA_OK) return st;
    if ((long long)B * H == 0) return LA_OK;
    PrefillArgs a = la::prefill_args(q, k, v, gamma_or_alpha, g, out, S_out, z_out, B, H, N, d, dv, &c);
    if (c.dtype == LA_BF16 && c.mode == LA_GLA) {
        // the GLA segment summaries have the kernelized modes' slot size
        if (N == 0) return la::write_start_state(a);
        const la::TcSegments sg = la::tc_segments_noalloc(B, H, N, d, dv);
        if (sg.G == 0) return LA_ERR_WORKSPACE;
        cudaError_t e;
        a.workspace = la::noalloc_scratch_address(&e);
        if (!a.workspace) return la::from_cuda(e);
        a.workspace_bytes = la::kNoAllocScratchBytes;
        return la::from_cuda(la::launch_prefill_tc_gla(a, sg));
    }
    if (!la::uses_tc_kernelized(c.dtype, c.mode)) {
        // paths that need no workspace run as la_prefill does; the bf16
        // gated delta rule's per-chunk operands grow with N and have no
        // fixed-size form
        if (la_prefill_workspace_bytes(B, H, N, d, dv, &c) != 0) return LA_ERR_UNSUPPORTED;
        return la::run_prefill(a);
    }
    if (N == 0) return la::write_start_state(a);
    if (la::tc_segments_noalloc(B, H, N, d, dv).G == 0) return LA_ERR_WORKSPACE;
    return la::from_cuda(la::launch_prefill_tc_kernelized_noalloc(a));
}

static la_status decode_common_checks(const void* q, const void* k, const void* v, float* S, void* out,
                                      int B, int H, int d, int dv, const la_config* cfg)
{
    if (!cfg) return LA_ERR_INVALID;
    if (B < 0 || H < 0) return LA_ERR_INVALID;
    if (cfg->dtype != LA_F32 && cfg->dtype != LA_BF16) return LA_ERR_INVALID;
    if (!la::head_ok(d) || !la::head_ok(dv)) return LA_ERR_UNSUPPORTED;
    if ((long long)B * H > 0 && (!q || !k || !v || !S || !out)) return LA_ERR_INVALID;
    if ((long long)B * H > 0x7fffffffLL) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

la_status la_decode_step(const void* q, const void* k, const void* v,
                         float* S, float* z, void* out,
                         int B, int H, int d, int dv, const la_config* cfg)
{
    la_status st = decode_common_checks(q, k, v, S, out, B, H, d, dv, cfg);
    if (st != LA_OK) return st;
    if (cfg->mode != LA_PLAIN) return LA_ERR_INVALID;
    if ((long long)B * H > 0 && !z) return LA_ERR_INVALID;
    if (!(cfg->eps >= 0.f)) return LA_ERR_INVALID;
    const void* ptrs[] = {q, k, v, S, z, out};
    for (const void* p : ptrs)
        if (!la::aligned16(p)) return LA_ERR_ALIGN;
    if ((long long)B * H == 0) return LA_OK;
    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.S = S; a.z = z; a.out = out;
    a.B = B; a.H = H; a.d = d; a.dv = dv; a.eps = cfg->eps; a.dtype = cfg->dtype;
    a.stream = static_cast<cudaStream_t>(cfg->stream);
    return la::from_cuda(la::launch_decode_kernelized(a));
}

la_status la_gated_delta_decode_step(const void* q, const void* k, const void* v,
                                     const float* alpha, const float* g,
                                     float* S, void* out,
                                     int B, int H, int d, int dv, const la_config* cfg)
{
    la_status st = decode_common_checks(q, k, v, S, out, B, H, d, dv, cfg);
    if (st != LA_OK) return st;
    if (cfg->mode != LA_GATED_DELTA) return LA_ERR_INVALID;
    if ((long long)B * H > 0 && (!alpha || !g)) return LA_ERR_INVALID;
    const void* ptrs[] = {q, k, v, alpha, g, S, out};
    for (const void* p : ptrs)
        if (!la::aligned16(p)) return LA_ERR_ALIGN;
    if ((long long)B * H == 0) return LA_OK;
    DecodeArgs a{};
    a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.g = g; a.S = S; a.out = out;
    a.B = B; a.H = H; a.d = d; a.dv = dv; a.dtype = cfg->dtype;
    a.stream = static_cast<cudaStream_t>(cfg->stream);
    return la::from_cuda(la::launch_decode_gated_delta(a));
}

la_status la_causal_conv(const void* x, const float* weight, const void* cache, void* out, void* cache_out,
                         int B, int H, int N, int d, int w, const la_config* cfg)
{
    if (!cfg) return LA_ERR_INVALID;
    if (B < 0 || H < 0 || N < 0 || w < 1) return LA_ERR_INVALID;
    if (cfg->dtype != LA_F32 && cfg->dtype != LA_BF16) return LA_ERR_INVALID;
    if (!la::head_ok(d) || w > 8) return LA_ERR_UNSUPPORTED;
    const long long chains = (long long)B * H;
    if (chains == 0) return LA_OK;
    if (N > 0 && (!x || !weight || !out)) return LA_ERR_INVALID;
    const size_t es = cfg->dtype == LA_BF16 ? 2 : 4;
    const size_t cache_bytes = (size_t)chains * (w - 1) * d * es;
    if (la::overlap(cache_out, cache_bytes, cache, cache_bytes) ||
        la::overlap(cache_out, cache_bytes, x, (size_t)chains * N * d * es))
        return LA_ERR_INVALID;
    const void* ptrs[] = {x, weight, cache, out, cache_out};
    for (const void* p : ptrs)
        if (!la::aligned16(p)) return LA_ERR_ALIGN;
    if (N == 0 && !cache_out) return LA_OK;
    la::ConvArgs a{};
    a.x = x; a.weight = weight; a.cache = cache; a.y = out; a.cache_out = w > 1 ? cache_out : nullptr;
    a.B = B; a.H = H; a.N = N; a.d = d; a.w = w;
    a.dtype = cfg->dtype;
    a.stream = static_cast<cudaStream_t>(cfg->stream);
    if (a.N == 0 && !a.cache_out) return LA_OK;
    return la::from_cuda(la::launch_causal_conv(a));
}

la_status la_set_stage_events(void* const* events, int n)
{
    if (n < 0 || n > la::kMaxStageEvents || (n > 0 && !events)) return LA_ERR_INVALID;
    for (int i = 0; i < n; ++i)
        if (!events[i]) return LA_ERR_INVALID;
    for (int i = 0; i < n; ++i) la::g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
    la::g_stage_count = n;
    return LA_OK;
}

la_status la_selftest_wait_timeout(void* stream)
{
    return la::from_cuda(la::launch_wait_timeout_selftest(static_cast<cudaStream_t>(stream)));
}

la_status la_prefill_check(const void* workspace, void* stream)
{
    (void)workspace;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LA_ERR_CUDA;
    const unsigned int e1 = la::read_and_clear_device_error(s);
    const unsigned int e2 = la::read_and_clear_device_error_gdelta(s);
    const unsigned int e3 = la::read_and_clear_device_error_selftest(s);
    const unsigned int e4 = la::read_and_clear_device_error_gla(s);
    if (e1 == 4u || e2 == 4u || e4 == 4u) return LA_ERR_UNSUPPORTED;
    if (e1 != 0 || e2 != 0 || e3 != 0 || e4 != 0) return LA_ERR_TIMEOUT;
    return LA_OK;
}

}  // extern "C"
