"""The C-ABI library loads, exports every symbol include/la.h declares, and
rejects bad arguments before launching anything (no GPU needed)."""
import ctypes
import os
import re

import pytest

import causal_kernelized_linear_la_b200 as la
from causal_kernelized_linear_la_b200 import LaConfig

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "la.h")


def declared():
    src = open(HEADER).read()
    return set(re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", src))


def test_header_declares_the_binding_exports():
    assert declared() == set(la.EXPORTS)


def test_binding_argument_counts_match_the_header():
    # every declared function is bound in Python with as many argument types
    # as the header gives it parameters
    src = open(HEADER).read()
    L = la.lib()
    for name, params in re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(([^)]*)\)", src):
        params = params.strip()
        n = 0 if params in ("", "void") else params.count(",") + 1
        assert len(getattr(L, name).argtypes) == n, name


def test_library_exports_every_declared_symbol():
    L = la.lib()
    for name in sorted(declared()):
        assert hasattr(L, name), name
    assert L.la_version().decode().count(".") == 2


def test_status_strings():
    for code in range(7):
        assert la.la_status_string(code).startswith("LA_")


def _cfg(dtype=la.LA_BF16, mode=0, eps=1e-6, S0=None, z0=None, ws=None, wsb=0):
    return LaConfig(dtype, mode, eps, None, S0, z0, ws, wsb)


FAKE = 0x10000  # never dereferenced: every call below fails validation first


def _prefill(cfg, B=1, H=1, N=8, d=64, dv=64, q=FAKE, k=FAKE, v=FAKE, ga=None, g=None, out=FAKE, S=FAKE, z=FAKE):
    c = ctypes.c_void_p
    return la.lib().la_prefill(c(q), c(k), c(v), c(ga), c(g), c(out), c(S), c(z), B, H, N, d, dv,
                               None if cfg is None else ctypes.byref(cfg))


def test_prefill_validation():
    assert _prefill(None) == la.LA_ERR_INVALID
    assert _prefill(_cfg(), B=-1) == la.LA_ERR_INVALID
    assert _prefill(_cfg(), d=96) == la.LA_ERR_UNSUPPORTED
    assert _prefill(_cfg(), dv=32) == la.LA_ERR_UNSUPPORTED
    assert _prefill(_cfg(dtype=7)) == la.LA_ERR_INVALID
    assert _prefill(_cfg(mode=9)) == la.LA_ERR_INVALID
    assert _prefill(_cfg(), q=FAKE + 8) == la.LA_ERR_ALIGN
    assert _prefill(_cfg(), S=0) == la.LA_ERR_INVALID
    assert _prefill(_cfg(), z=0) == la.LA_ERR_INVALID                  # kernelized needs z_out
    assert _prefill(_cfg(mode=2), ga=FAKE, g=FAKE) == la.LA_ERR_INVALID  # delta must not get z_out
    assert _prefill(_cfg(mode=1)) == la.LA_ERR_INVALID                  # decay needs gamma
    assert _prefill(_cfg(mode=0), ga=FAKE) == la.LA_ERR_INVALID         # plain takes no gamma
    assert _prefill(_cfg(eps=-1.0)) == la.LA_ERR_INVALID
    assert _prefill(_cfg(S0=FAKE), S=FAKE) == la.LA_ERR_INVALID          # output aliases start state
    # partial overlaps are rejected too (S0 spans 64*64*4 bytes from FAKE)
    assert _prefill(_cfg(S0=FAKE), S=FAKE + 4096) == la.LA_ERR_INVALID
    assert _prefill(_cfg(S0=FAKE), S=FAKE - 4096) == la.LA_ERR_INVALID
    assert _prefill(_cfg(S0=FAKE), S=FAKE + (1 << 20), z=FAKE + 256) == la.LA_ERR_INVALID
    assert _prefill(_cfg(z0=FAKE + 16384 - 16), S=FAKE) == la.LA_ERR_INVALID
    # nothing to do: valid and launches nothing
    assert _prefill(_cfg(), B=0) == la.LA_OK
    assert _prefill(_cfg(), H=0, q=0, k=0, v=0, out=0, S=0, z=0) == la.LA_OK


def test_decode_validation():
    c = ctypes.c_void_p
    L = la.lib()
    cfg = _cfg()
    assert L.la_decode_step(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), 1, 1, 64, 48, ctypes.byref(cfg)) == la.LA_ERR_UNSUPPORTED
    assert L.la_decode_step(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(0), c(FAKE), 1, 1, 64, 64, ctypes.byref(cfg)) == la.LA_ERR_INVALID
    assert L.la_decode_step(c(FAKE + 4), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), 1, 1, 64, 64, ctypes.byref(cfg)) == la.LA_ERR_ALIGN
    dcfg = _cfg(mode=2)
    assert L.la_decode_step(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), 1, 1, 64, 64, ctypes.byref(dcfg)) == la.LA_ERR_INVALID
    assert L.la_gated_delta_decode_step(c(FAKE), c(FAKE), c(FAKE), c(0), c(FAKE), c(FAKE), c(FAKE), 1, 1, 64, 64, ctypes.byref(dcfg)) == la.LA_ERR_INVALID
    assert L.la_gated_delta_decode_step(c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), c(FAKE), 0, 4, 64, 64, ctypes.byref(dcfg)) == la.LA_OK


def test_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64)
    with pytest.raises(ValueError):
        la.la_prefill(q, q, q)
    with pytest.raises(ValueError, match="CUDA"):
        la.la_prefill_varlen(q, q, q, [5])


def test_varlen_binding_checks_the_lengths_list():
    import torch
    q = torch.zeros(2, 1, 8, 64)
    with pytest.raises(ValueError, match="seq_lens"):
        la.la_prefill_varlen(q, q, q, [5])            # one length for a batch of two
    with pytest.raises(ValueError, match="mode"):
        la.la_prefill_varlen(q, q, q, [5, 8], mode="softmax")


def test_workspace_query_is_host_only():
    n = la.la_prefill_workspace_bytes(2, 16, 32768, 128, 128, "bf16", "decay")
    assert n >= 0


def test_gated_delta_workspace_size():
    # bf16 gated delta: per chain ceil(N/64)*64 rows of d + 128 bf16 values and
    # two fp32 factors per token; f32 needs none
    n = la.la_prefill_workspace_bytes(1, 32, 1000, 128, 128, "bf16", "gated_delta")
    assert n == 32 * (1024 * (128 + 128) * 2 + 1024 * 2 * 4)
    assert la.la_prefill_workspace_bytes(1, 32, 1000, 128, 128, "f32", "gated_delta") == 0
    # the long workload runs as eight parts (whole chunks of 64 tokens, 65536 in
    # all), plus two carry states
    part = 32 * (8192 * (128 + 128) * 2 + 8192 * 2 * 4)
    n = la.la_prefill_workspace_bytes(1, 32, 65536, 128, 128, "bf16", "gated_delta")
    assert n == 8 * part + 2 * 32 * 128 * 128 * 4


def test_gated_delta_parts_are_whole_chunks():
    """Long gated-delta sequences run as growing parts; every part but the last
    is whole 64-token chunks, so the parts' workspace slices add up to the
    workspace of the whole padded sequence (a ragged middle part would pad
    itself), plus the two carry states (host-only query)."""
    for B, H, N, d in ((1, 2, 9000, 128), (1, 2, 12345, 64), (1, 32, 65536, 128), (1, 4, 100000, 128),
                       (2, 8, 8192, 64)):
        chains, nch = B * H, -(-N // 64)
        one = chains * (nch * 64 * (d + 128) * 2 + nch * 2 * 64 * 4)
        parts = la.la_prefill_kernel_count(B, H, N, d, d, "bf16", "gated_delta") // 2
        assert parts == min(8, nch // 32), (N, d, parts)
        carries = 2 * chains * d * d * 4 if parts > 1 else 0
        got = la.la_prefill_workspace_bytes(B, H, N, d, d, "bf16", "gated_delta")
        assert got == one + carries, (B, H, N, d, got, one + carries)


def test_kernel_count():
    kc = la.la_prefill_kernel_count
    assert kc(4, 8, 4096, 64, 64, "bf16", "plain") == 3
    assert kc(2, 16, 32768, 128, 128, "bf16", "decay") == 3
    assert kc(1, 32, 65536, 128, 128, "bf16", "gated_delta") == 16    # eight overlapped parts
    assert kc(1, 32, 8192, 128, 128, "bf16", "gated_delta") == 8      # four parts
    assert kc(1, 3, 2100, 128, 128, "bf16", "gated_delta") == 2
    assert kc(64, 32, 65536, 128, 128, "bf16", "gated_delta") == 2    # enough chains to fill the GPU
    assert kc(1, 1, 256, 64, 64, "f32", "plain") == 2        # parallel form: outputs, final state
    assert kc(1, 1, 5000, 64, 64, "f32", "plain") == 1       # chunk loop
    assert kc(1, 32, 8192, 128, 128, "bf16", "gla") == 3      # summaries, scan, chunk loop
    assert kc(1, 32, 8192, 128, 128, "f32", "gla") == 1
    assert kc(1, 1, 0, 64, 64, "bf16", "plain") == 0


def test_stage_events_validation():
    # host-only: argument checks of the profiling hook, no CUDA call is made
    L = la.lib()
    c = ctypes.c_void_p
    assert L.la_set_stage_events(None, 1) == la.LA_ERR_INVALID
    arr = (c * 1)(c(0))
    assert L.la_set_stage_events(arr, 1) == la.LA_ERR_INVALID      # NULL handle
    assert L.la_set_stage_events(arr, 17) == la.LA_ERR_INVALID     # more than 16
    assert L.la_set_stage_events(None, -1) == la.LA_ERR_INVALID
    assert L.la_set_stage_events(None, 0) == la.LA_OK              # off


def test_conv_validation_host_only():
    # argument checks of la_causal_conv that return before any CUDA call
    L = la.lib()
    c = ctypes.c_void_p
    cfg = LaConfig(la.LA_BF16, 0, 0.0, None, None, None, None, 0)
    FAKE = c(1 << 20)   # never dereferenced: every call below fails validation first
    assert L.la_causal_conv(FAKE, FAKE, None, FAKE, None, 1, 1, 8, 64, 0, ctypes.byref(cfg)) == la.LA_ERR_INVALID
    assert L.la_causal_conv(FAKE, FAKE, None, FAKE, None, 1, 1, 8, 64, 9, ctypes.byref(cfg)) == la.LA_ERR_UNSUPPORTED
    assert L.la_causal_conv(FAKE, FAKE, None, FAKE, None, 1, 1, 8, 32, 4, ctypes.byref(cfg)) == la.LA_ERR_UNSUPPORTED
    assert L.la_causal_conv(None, FAKE, None, FAKE, None, 1, 1, 8, 64, 4, ctypes.byref(cfg)) == la.LA_ERR_INVALID
    # cache_out overlapping the cache
    assert L.la_causal_conv(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 8, 64, 4, ctypes.byref(cfg)) == la.LA_ERR_INVALID
    # misaligned pointer
    assert L.la_causal_conv(c((1 << 20) + 2), FAKE, None, FAKE, None, 1, 1, 8, 64, 4, ctypes.byref(cfg)) == la.LA_ERR_ALIGN
    # nothing to do
    assert L.la_causal_conv(None, None, None, None, None, 0, 4, 8, 64, 4, ctypes.byref(cfg)) == la.LA_OK


def _varlen(cfg, lens, B=2, H=1, N=8, d=64, dv=64, q=FAKE, out=FAKE, S=FAKE, z=FAKE):
    c = ctypes.c_void_p
    arr = None if lens is None else (ctypes.c_int * len(lens))(*lens)
    return la.lib().la_prefill_varlen(c(q), c(q), c(q), None, None, c(out), c(S), c(z), arr, B, H, N, d, dv,
                                      ctypes.byref(cfg))


def test_varlen_validation():
    # every call fails validation before anything is launched
    assert _varlen(_cfg(), [3, 9]) == la.LA_ERR_INVALID        # a length past the padded N
    assert _varlen(_cfg(), [-1, 2]) == la.LA_ERR_INVALID       # negative length
    assert _varlen(_cfg(), None) == la.LA_ERR_INVALID          # lengths missing
    assert _varlen(_cfg(), [3, 8], q=FAKE + 4) == la.LA_ERR_ALIGN
    assert _varlen(_cfg(), [3, 8], d=48) == la.LA_ERR_UNSUPPORTED
    assert _varlen(_cfg(), [3, 8], z=0) == la.LA_ERR_INVALID   # kernelized modes need z_out
    assert _varlen(_cfg(), None, B=0) == la.LA_OK              # nothing to do
    # bf16 kernelized needs a workspace for its segment summaries
    assert _varlen(_cfg(), [3, 8]) == la.LA_ERR_WORKSPACE


def test_varlen_workspace_is_one_slice_per_sequence():
    # paths that run one sequence at a time take one 256-byte aligned slice each
    lens = [0, 100, 5000, 64, 4096]
    for dtype, mode in (("bf16", "gated_delta"), ("f32", "plain"), ("bf16", "gla")):
        each = [la.la_prefill_workspace_bytes(1, 8, n, 128, 128, dtype, mode) if n > 0 else 0 for n in lens]
        want = sum((n + 255) // 256 * 256 for n in each)
        assert la.la_prefill_varlen_workspace_bytes(lens, 8, 128, 128, dtype, mode) == want
    assert la.la_prefill_varlen_workspace_bytes([], 8, 128, 128) == 0


def _one_set_units(lens, H, d, dv):
    """Segments of the one-launch-set padded batch: the smallest segment length
    (a multiple of 64 tokens, at least 128, at most 4096) whose segment count
    over all (sequence, head) chains fits one wave of resident CTAs."""
    slots = 296 if (d, dv) == (64, 64) else 148
    L = 128
    while True:
        units = sum(H * -(-n // L) for n in lens)
        if units <= slots or L >= 4096:
            return L, units
        L += 64


def test_varlen_workspace_of_the_one_launch_set():
    # the bf16 kernelized modes run a padded batch as one launch set; its
    # workspace holds one (d*dv + d) fp32 summary per segment
    cases = [([0, 100, 5000, 64, 4096], 8, 128, 128), ([1] * 64, 32, 64, 64),
             ([65536, 3, 0], 16, 128, 64), ([0, 0], 4, 64, 128)]
    for lens, H, d, dv in cases:
        L, units = _one_set_units(lens, H, d, dv)
        assert L % 64 == 0 and 128 <= L <= 4096
        for mode in ("plain", "decay"):
            got = la.la_prefill_varlen_workspace_bytes(lens, H, d, dv, "bf16", mode)
            assert got == units * (d * dv + d) * 4, (lens, H, d, dv, mode)
    # more sequences than one launch set takes: one slice per sequence again
    lens = [100] * 65
    each = la.la_prefill_workspace_bytes(1, 8, 100, 64, 64, "bf16", "plain")
    want = 65 * ((each + 255) // 256 * 256)
    assert la.la_prefill_varlen_workspace_bytes(lens, 8, 64, 64, "bf16", "plain") == want
