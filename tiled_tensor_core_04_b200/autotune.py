"""Per-shape choice of tile configuration and cache hints by measurement.

The planner in the library picks a tiling from a wave-count cost model.  This
module instead times a small set of alternatives on the device and keeps the
fastest for each problem shape:
- the planner's own choice;
- the three CTA-pair tile widths and the 1-CTA tile;
- swizzle panels of 4 and 16 tile rows;
- L2 eviction hints on the operand loads;
- for skinny M, the split-K / stream-K settings of the swap-AB kernel.

The TileLang notes leave tile sizes, pipeline depth and the swizzle panel to
the user or an autotuner.  The Ascend variant adds L2 cache-control hints.

Every candidate is a `gemm_relu_options_t` setting covered by the parity tests;
this module only measures them and adds no arithmetic of its own.
"""
from __future__ import annotations

import json
import statistics

from . import _abi

# Knobs that change what the kernel does without changing the plan.
RUNTIME_KNOBS = ("l2_hint_a", "l2_hint_b", "c_streaming", "wait_sleep_ns")

_CACHE: dict[tuple, dict | None] = {}
tune_calls = 0  # number of measurements made (tests check the cache with it)


def candidates(M, N, K, in_dtype, out_dtype, trans_b, num_sms=148) -> list[dict | None]:
    """Option settings worth timing for this shape, the planner's choice first.
    Settings whose plan and runtime knobs equal an earlier one are dropped."""
    cands: list[dict | None] = [None]
    if M > 64:
        for wide in (2, 1) + ((3,) if trans_b else ()):
            cands.append({"cta_pair": _abi.GEMM_CTA_PAIR, "wide": wide})
        cands.append({"cta_pair": _abi.GEMM_CTA_SINGLE})
        cands += [{"panel": 4}, {"panel": 16}, {"l2_hint_a": 2}, {"l2_hint_a": 2, "l2_hint_b": 1}]
    if M <= 128:
        cands += [{"swap_ab": 1, "split_k": s} for s in (1, 2, 4, 8)]
        cands.append({"swap_ab": 1, "stream_k": 1})
    out, seen = [], set()
    for o in cands:
        try:
            plan = _abi.gemm_relu_plan(M, N, K, in_dtype, out_dtype, trans_b, num_sms=num_sms,
                                       options=o)
        except _abi.GemmError:
            continue
        knobs = {k: v for k, v in (o or {}).items() if k in RUNTIME_KNOBS}
        key = json.dumps([plan, knobs], sort_keys=True)
        if key not in seen:
            seen.add(key)
            out.append(o)
    return out


def tune(A, B, C, M, N, K, in_dtype, out_dtype, trans_b, relu=True, stream=None, iters=10,
         warmup=3, flush_bytes=0, cands=None):
    """Times every candidate (median of `iters` calls after `warmup`, CUDA events on the
    call's stream, optionally writing `flush_bytes` between calls to empty L2) and returns
    (best options, [(options, median ms), ...]).  C is overwritten."""
    import torch

    global tune_calls
    dev = torch.cuda.current_device()
    if cands is None:
        cands = candidates(M, N, K, in_dtype, out_dtype, trans_b,
                           torch.cuda.get_device_properties(dev).multi_processor_count)
    s = torch.cuda.current_stream() if stream is None else stream
    flush = torch.empty(flush_bytes, dtype=torch.uint8, device=dev) if flush_bytes else None
    table = []
    for o in cands:
        def call():
            _abi.gemm_relu_ex(A, B, C, M, N, K, in_dtype, out_dtype, trans_b, relu, s.cuda_stream,
                              options=o)
        with torch.cuda.stream(s):
            for _ in range(warmup):
                call()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(iters)]
            for e0, e1 in ev:
                if flush is not None:
                    flush.fill_(1)
                e0.record(s)
                call()
                e1.record(s)
        s.synchronize()
        table.append((o, statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)))
        tune_calls += 1
    st, detail = _abi.gemm_relu_last_device_error()
    if st != _abi.GEMM_OK:
        raise _abi.GemmError(st, f"a bounded device wait ran out while tuning (bits {detail:#x})")
    best = min(table, key=lambda t: t[1])
    return best[0], table


def tuned_options(A, B, C, M, N, K, in_dtype, out_dtype, trans_b, relu=True, stream=None,
                  **kw):
    """The fastest options for this problem shape on this device, measured once per
    process and cached (C is overwritten by the measurement)."""
    import torch

    key = (int(M), int(N), int(K), _abi._dtype(in_dtype), _abi._dtype(out_dtype),
           bool(trans_b), bool(relu), torch.cuda.get_device_name())
    if key not in _CACHE:
        _CACHE[key] = tune(A, B, C, M, N, K, in_dtype, out_dtype, trans_b, relu, stream, **kw)[0]
    return _CACHE[key]
