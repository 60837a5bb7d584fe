"""Cycle trace of the forward kernel, from the ATTN_TRACE build of the library.

    python -m exact_attention_145_b200.trace --workload causal_gqa_llama8b_s2048

Builds libattn_trace.so (the same kernels with trace records at the pipeline
hand-offs), runs the workload a few times, keeps the records of the last
launch and prints one JSON summary: per key step of each softmax subtile the
cycles spent waiting for S, in the softmax (S ready -> P handed over) and
between handing P over and the next S (the PV and next QK^T on the tensor
pipe plus the wake-ups); the prologue (kernel start -> first S), the unit
boundaries (last P of a unit -> first S of the next), the epilogue, and the
longest CTA's total. Times are SM cycles (clock64), medians over CTAs and
steps unless stated. Trace records cost a few cycles each, so absolute times
run slightly above the untraced kernel's.
"""
from __future__ import annotations

import argparse
import json
import os
import sys

import numpy as np

ROLES = tuple("softmax%d.w%d" % (w // 4, w) for w in range(8)) + ("mma0", "tma", "mma1")
N_ROLES = len(ROLES)
MMA_ROLES, TMA = (8, 10), 9
MMA = MMA_ROLES[0]
EV = dict(S_WAIT=1, S_READY=2, P_DONE=3, O_WAIT=4, EPI_BEGIN=5, EPI_END=6, Q_FULL=10, PV=11, QK=12, P_WAIT=13,
          MMA_END=14, PV_ISSUED=15, Q_LOAD=20, KV_LOAD=21, KERNEL_END=30)


def decode_records(raw: np.ndarray, grid: int, per_role: int):
    """raw: uint32 [grid, roles, per_role, 2] -> per CTA, per role, list of (cycle, event, aux)."""
    out = []
    for c in range(grid):
        roles = []
        for r in range(raw.shape[1]):
            rec = raw[c, r]
            n = int(np.count_nonzero(rec[:, 1]))
            roles.append([(int(t), int(x) >> 24, int(x) & 0xFFFFFF) for t, x in rec[:n]])
        out.append(roles)
    return out


def _med(x):
    return float(np.median(x)) if len(x) else None


def summarize(ctas) -> dict:
    soft_full, soft_part, s_wait, ret, period = [], [], [], [], []
    prologue, boundary, epi, o_wait, kend = [], [], [], [], []
    pv_wait = []
    skew = []
    per_cta = []
    for roles in ctas:
        end = [t for t, e, _ in roles[0] if e == EV["KERNEL_END"]]
        kend.append(end[0] if end else 0)
        for s in (0, 1):
            recs = roles[4 * s]
            last_p, first_s_of_unit, unit_idx = None, True, 0
            prev_ready = None
            for i, (t, e, aux) in enumerate(recs):
                if e == EV["S_WAIT"]:
                    wait_t = t
                elif e == EV["S_READY"]:
                    s_wait.append(t - wait_t)
                    if first_s_of_unit:
                        if unit_idx == 0 and s == 0:
                            prologue.append(t)
                        elif last_p is not None:
                            boundary.append(t - last_p)
                        first_s_of_unit = False
                        prev_ready = None
                    elif last_p is not None:
                        ret.append(t - last_p)
                    if prev_ready is not None:
                        period.append(t - prev_ready)
                    prev_ready = t
                    ready_t, cls = t, aux >> 20
                elif e == EV["P_DONE"]:
                    (soft_full if cls == 2 else soft_part).append(t - ready_t)
                    last_p = t
                elif e == EV["O_WAIT"]:
                    o_wait_t = t
                elif e == EV["EPI_BEGIN"]:
                    o_wait.append(t - o_wait_t)
                    epi_t = t
                elif e == EV["EPI_END"]:
                    epi.append(t - epi_t)
                    first_s_of_unit, unit_idx = True, unit_idx + 1
        mma = [x for r in MMA_ROLES if r < len(roles) for x in roles[r]]
        # skew: per step, last warp of a subtile to hand over P minus the first
        for sub in (0, 1):
            done = {}
            for w in range(4 * sub, 4 * sub + 4):
                for t, e, aux in roles[w] if w < len(roles) else []:
                    if e == EV["P_DONE"]:
                        done.setdefault(aux, []).append(t)
            skew.extend(max(v) - min(v) for v in done.values() if len(v) == 4)
        waits = {}
        for t, e, aux in mma:
            if e == EV["P_WAIT"]:
                waits[aux] = t
            elif e == EV["PV"] and aux in waits:
                pv_wait.append(t - waits.pop(aux))
        steps0 = sum(1 for _, e, _ in roles[0] if e == EV["S_READY"])
        units0 = sum(1 for _, e, _ in roles[0] if e == EV["EPI_END"])
        per_cta.append((end[0] if end else 0, steps0, units0))
    crit = max(per_cta) if per_cta else (0, 0, 0)
    return {
        "ctas": len(ctas),
        "kernel_cycles_max": int(max(kend)) if kend else None,
        "kernel_cycles_median": _med(kend),
        "critical_cta": {"cycles": crit[0], "steps": crit[1], "units": crit[2]},
        "softmax_full_tile": _med(soft_full), "softmax_partial_tile": _med(soft_part),
        "s_wait": _med(s_wait), "p_to_next_s": _med(ret), "step_period_per_subtile": _med(period),
        "prologue_to_first_s": _med(prologue), "unit_boundary": _med(boundary),
        "o_wait_before_epilogue": _med(o_wait), "epilogue": _med(epi),
        "mma_wait_for_p": _med(pv_wait),
        "p_handover_skew_across_warps": _med(skew),
        "counts": {"full_steps": len(soft_full), "partial_steps": len(soft_part), "boundaries": len(boundary)},
    }


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="causal_gqa_llama8b_s2048")
    ap.add_argument("--launches", type=int, default=4)
    ap.add_argument("--per-role", type=int, default=512)
    ap.add_argument("--save", default=None, help="write the raw records (.npy) here")
    args = ap.parse_args(argv)
    os.environ["ATTN_LIBRARY_VARIANT"] = "trace"
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    from . import build as _build
    _build.build(trace=True)
    import torch

    from . import _lib, attn_build_block_mask, attn_fwd
    import workloads as W
    lib = _lib.load()
    if not hasattr(lib, "attn_trace_configure"):
        raise RuntimeError("loaded library is not the trace build")
    w = W.WORKLOADS[args.workload]
    d = W.make_prefill_inputs(w)
    dev = torch.device("cuda", 0)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    q, k, v = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    kw = {}
    if w.mask == W.MASK_CAUSAL:
        kw["causal"] = True
    elif w.mask == W.MASK_WINDOW:
        kw["window"] = (w.window_left, w.window_right)
    elif w.mask == W.MASK_DOCUMENT:
        kw["doc_id"] = torch.from_numpy(d["doc_id"]).to(dev)
        kw["block_mask"] = attn_build_block_mask(w.S, w.S, doc_id=kw["doc_id"])
    if w.mod == W.MOD_SOFTCAP:
        kw["softcap"] = w.softcap
    elif w.mod == W.MOD_ALIBI:
        kw["alibi_slopes"] = torch.from_numpy(d["alibi"]).to(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    buf = torch.zeros((sms, N_ROLES, args.per_role, 2), dtype=torch.int32, device=dev)
    for i in range(args.launches):
        buf.zero_()
        _lib.check(lib.attn_trace_configure(buf.data_ptr(), args.per_role), "attn_trace_configure")
        attn_fwd(q, k, v, **kw)
        torch.cuda.synchronize()
    _lib.check(lib.attn_trace_configure(None, 0), "attn_trace_configure")
    raw = buf.cpu().numpy().view(np.uint32)
    grid = int(np.count_nonzero(raw[:, 0, 0, 1] != 0))
    if args.save:
        np.save(args.save, raw[:grid])
    summary = summarize(decode_records(raw, grid, args.per_role))
    summary["workload"] = w.name
    print(json.dumps(summary))
    return 0


if __name__ == "__main__":
    sys.exit(main())
