"""Event timelines of one CTA, recorded by the debug build of the library.

The debug build (``python -m exact_io_aware_tmem_b200.build --debug``,
libfa_b200_debug.so) stamps the SM clock at the events of each role of the
traced CTA: waits passed, products issued, signals sent, one stamp per step
(include/fa.h, "Debug build"). This module runs one pass of a kernel on a
workload through that build and reports, over the steady-state steps, the
median number of cycles between the events: where each role waits, and for
what.

  python -m exact_io_aware_tmem_b200.trace --kernel bwd --workload NAME [--cta 0]
  python -m exact_io_aware_tmem_b200.trace --kernel fwd --workload NAME
  python -m exact_io_aware_tmem_b200.trace --kernel dec --workload DECODE_NAME
  python -m exact_io_aware_tmem_b200.trace --kernel d64 --workload bf16_fwd_b4_h16_n2048_d64

The balanced decode and the D = 64 forward also record every CTA's SM and
global-timer span (the first 1024 CTAs): how long CTAs take, and how much of
each SM's time they cover.

The traced CTA is blockIdx.x (0: the first launched, with the longest causal
work).
"""
from __future__ import annotations

import argparse
import statistics
import sys

import numpy as np

# Event kinds, as numbered in the kernels' sources.
BWD_KINDS = {
    "P_Q": 0, "P_DO": 1, "M_PREADY": 2, "M_SNEXT": 3, "M_DSREADY": 4, "M_DQ": 5,
    "M_DQFREE": 6, "M_DP": 7, "S_SFULL": 8, "S_PREADY": 9, "Q_DQFULL": 10, "Q_DQFREE": 11,
    "Q_STAGED": 12, "S_DPFULL": 13, "S_DSREADY": 14, "M_DV": 15, "S_SLD": 16, "S_EXPD": 17,
    "S_DPLD": 18, "S_DSC": 19, "S_DSST": 20,
}
FWD_KINDS = {
    "P_K": 0, "P_V": 1, "M_VFULL": 2, "M_PV0": 3, "M_S0": 4, "M_PV1": 5, "M_S1": 6,
    "W0_SFULL": 7, "W0_LD": 8, "W0_EXP": 9, "W0_ARR": 10,
    "W1_SFULL": 11, "W1_LD": 12, "W1_EXP": 13, "W1_ARR": 14,
    "M_PREADY0": 15, "M_PREADY1": 16,
}
DEC_KINDS = {
    "P_K": 0, "P_V": 1, "M_S": 2, "M_PV": 3, "W_SFULL": 4, "W_ARR": 5, "W_EPI": 6,
}
D64_KINDS = {
    "W_SFULL": 0, "W_LD": 1, "W_EXP": 2, "W_ARR": 3, "M_S": 4, "M_PV": 5, "W_EPI": 6,
}
# (label, from event, step offset of from, to event, step offset of to): the
# median of stamp[to][t + dto] - stamp[from][t + dfrom] over the steps t.
BWD_SPANS = [
    ("dS warps: exponentials of S_t (s_full -> p_ready)", "S_SFULL", 0, "S_PREADY", 0),
    ("  first 32 scores in registers", "S_SFULL", 0, "S_SLD", 0),
    ("  -> exponentials of 64 scores done", "S_SLD", 0, "S_EXPD", 0),
    ("  -> P in TMEM, p_ready", "S_EXPD", 0, "S_PREADY", 0),
    ("dS warps: wait for dP_t (p_ready -> dp_full)", "S_PREADY", 0, "S_DPFULL", 0),
    ("dS warps: dS phase (dp_full -> ds_ready)", "S_DPFULL", 0, "S_DSREADY", 0),
    ("  first 32 of dP in registers", "S_DPFULL", 0, "S_DPLD", 0),
    ("  -> dS of 64 formed", "S_DPLD", 0, "S_DSC", 0),
    ("  -> dS to shared memory", "S_DSC", 0, "S_DSST", 0),
    ("  -> fences, ds_ready", "S_DSST", 0, "S_DSREADY", 0),
    ("dS warps: wait for S_{t+1} (ds_ready -> s_full)", "S_DSREADY", 0, "S_SFULL", 1),
    ("step period (s_full -> s_full)", "S_SFULL", 0, "S_SFULL", 1),
    ("dQ warps: read-out of dQ_t (dq_full -> dq_free)", "Q_DQFULL", 0, "Q_DQFREE", 0),
    ("dQ warps: staged, reductions issued (dq_free -> staged)", "Q_DQFREE", 0, "Q_STAGED", 0),
    ("MMA: p_ready seen after arrival", "S_PREADY", 0, "M_PREADY", 0),
    ("MMA: dV_t issued (p_ready seen -> issued)", "M_PREADY", 0, "M_DV", 0),
    ("MMA: S_{t+1} issued after dV_t", "M_DV", 0, "M_SNEXT", 1),
    ("MMA: ds_ready seen after arrival", "S_DSREADY", 0, "M_DSREADY", 0),
    ("MMA: dQ_t issued (ds_ready seen -> dQ issued)", "M_DSREADY", 0, "M_DQ", 0),
    ("MMA: dq_free seen after arrival", "Q_DQFREE", 0, "M_DQFREE", 0),
    ("MMA: dP_{t+1} issued after dq_free", "M_DQFREE", 0, "M_DP", 1),
    ("tensor: S_{t+1} issue -> s_full seen", "M_SNEXT", 1, "S_SFULL", 1),
    ("tensor: dQ_t issue -> dq_full seen", "M_DQ", 0, "Q_DQFULL", 0),
    ("tensor: dP_{t+1} issue -> dp_full seen", "M_DP", 1, "S_DPFULL", 1),
    ("producer: Q_{t+1} issued before S_{t+1} issue", "P_Q", 1, "M_SNEXT", 1),
    ("producer: dO_{t+1} issued before dP_{t+1} issue", "P_DO", 1, "M_DP", 1),
]
FWD_SPANS = [
    ("group 0: load S (s_full -> scores in registers)", "W0_SFULL", 0, "W0_LD", 0),
    ("group 0: max, exponentials, P stored (-> exp done)", "W0_LD", 0, "W0_EXP", 0),
    ("group 0: rescale, P visible (-> p_ready)", "W0_EXP", 0, "W0_ARR", 0),
    ("group 0: wait for next scores (p_ready -> s_full)", "W0_ARR", 0, "W0_SFULL", 1),
    ("group 0: tile period", "W0_SFULL", 0, "W0_SFULL", 1),
    ("group 1: load S", "W1_SFULL", 0, "W1_LD", 0),
    ("group 1: max, exponentials, P stored", "W1_LD", 0, "W1_EXP", 0),
    ("group 1: rescale, P visible", "W1_EXP", 0, "W1_ARR", 0),
    ("group 1: wait for next scores", "W1_ARR", 0, "W1_SFULL", 1),
    ("group 1: tile period", "W1_SFULL", 0, "W1_SFULL", 1),
    ("group 1 start after group 0 start", "W0_SFULL", 0, "W1_SFULL", 0),
    ("MMA: p_ready(0) seen after arrival", "W0_ARR", 0, "M_PREADY0", 0),
    ("MMA: P_0 V_j issued", "M_PREADY0", 0, "M_PV0", 0),
    ("MMA: S_0 of j+1 issued after P_0 V_j", "M_PV0", 0, "M_S0", 1),
    ("MMA: p_ready(1) seen after arrival", "W1_ARR", 0, "M_PREADY1", 0),
    ("MMA: wait for p_ready(1) after S_0 issue", "M_S0", 1, "M_PREADY1", 0),
    ("tensor: S_0 issue -> s_full seen by group 0", "M_S0", 1, "W0_SFULL", 1),
    ("tensor: S_1 issue -> s_full seen by group 1", "M_S1", 1, "W1_SFULL", 1),
    ("producer: K_{j+1} issued before S_0 of j+1 issue", "P_K", 1, "M_S0", 1),
    ("producer: V_j issued before the MMA saw it", "P_V", 0, "M_VFULL", 0),
]


# Per-CTA records of the balanced decode (index = CTA): SM + 1, and the
# global timer (ns) at the CTA's start and end.

DEC_SPANS = [
    ("producer: K_j issued -> S_j issued (K landed, S buffer free)", "P_K", 0, "M_S", 0),
    ("tensor: S_j issued -> softmax sees S_j", "M_S", 0, "W_SFULL", 0),
    ("softmax: S_j seen -> P_j published", "W_SFULL", 0, "W_ARR", 0),
    ("MMA warp: P_j published -> P_j V_j issued", "W_ARR", 0, "M_PV", 0),
    ("softmax: tile period (P_j -> P_{j+1} published)", "W_ARR", 0, "W_ARR", 1),
    ("MMA warp: tile period (P_j V_j -> P_{j+1} V_{j+1})", "M_PV", 0, "M_PV", 1),
    ("producer: K_j issue period", "P_K", 0, "P_K", 1),
    ("producer: V_j issue period", "P_V", 0, "P_V", 1),
    ("producer: K_{j+3} issued after S_j issued (slot refill)", "M_S", 0, "P_K", 3),
    ("producer: V_{j+3} issued after P_j V_j issued (slot refill)", "M_PV", 0, "P_V", 3),
]


D64_SPANS = [
    ("softmax: S_j seen -> scores in registers", "W_SFULL", 0, "W_LD", 0),
    ("softmax: scores in registers -> exponentials done", "W_LD", 0, "W_EXP", 0),
    ("softmax: exponentials done -> P_j published", "W_EXP", 0, "W_ARR", 0),
    ("softmax: P_j published -> S_{j+1} seen", "W_ARR", 0, "W_SFULL", 1),
    ("softmax: tile period (S_j seen -> S_{j+1} seen)", "W_SFULL", 0, "W_SFULL", 1),
    ("MMA warp: scores of S_j read -> S_{j+1} issued", "W_LD", 0, "M_S", 1),
    ("tensor: S_j issued -> softmax sees S_j", "M_S", 0, "W_SFULL", 0),
    ("MMA warp: P_j published -> P_j V_j issued", "W_ARR", 0, "M_PV", 0),
]
CTA_SM, CTA_START, CTA_END = 29, 30, 31


def cta_report(stamps) -> list:
    """Lines on the CTAs' global-timer spans: count, durations, and per SM the
    CTA time over the wall time (mean CTAs resident) and the share of the
    wall time with at least one CTA resident."""
    st = stamps[CTA_START].astype(np.int64)
    en = stamps[CTA_END].astype(np.int64)
    sm = stamps[CTA_SM].astype(np.int64) - 1
    ok = (st != 0) & (en != 0) & (sm >= 0)
    if not ok.any():
        return []
    st, en, sm = st[ok], en[ok], sm[ok]
    t0, t1 = st.min(), en.max()
    wall = max(int(t1 - t0), 1)
    dur = (en - st) / 1e3
    lines = [f"  CTAs: {int(ok.sum())}, all done {wall / 1e3:.1f} us after the first started; "
             f"start spread {(st.max() - t0) / 1e3:.1f} us; duration min {dur.min():.1f} "
             f"median {np.median(dur):.1f} max {dur.max():.1f} us"]
    resident, covered = [], []
    for s in np.unique(sm):
        a, b = st[sm == s], en[sm == s]
        resident.append(float((b - a).sum()) / wall)
        ev = sorted([(int(x), 1) for x in a] + [(int(y), -1) for y in b])
        live, last, cov = 0, int(t0), 0
        for t, d in ev:
            if live > 0:
                cov += t - last
            live += d
            last = t
        covered.append(cov / wall)
    lines.append(f"  SMs: {len(resident)}; mean CTAs resident {statistics.fmean(resident):.2f} "
                 f"(min {min(resident):.2f}); time with a CTA resident "
                 f"{100 * statistics.fmean(covered):.1f} % (min {100 * min(covered):.1f} %)")
    return lines


def spans(stamps, kinds: dict, table, n_steps: int, skip: int = 2) -> list:
    """(label, median, mean, 90th percentile cycles, count) for each span of
    ``table``."""
    out = []
    for label, a, da, b, db in table:
        d = []
        for t in range(skip, n_steps - skip):
            ta, tb = t + da, t + db
            if not (0 <= ta < 1024 and 0 <= tb < 1024):
                continue
            x, y = int(stamps[kinds[a]][ta]), int(stamps[kinds[b]][tb])
            if x and y:
                d.append(y - x)
        if d:
            d.sort()
            out.append((label, statistics.median(d), statistics.fmean(d),
                        d[min(len(d) - 1, int(0.9 * len(d)))], len(d)))
        else:
            out.append((label, None, None, None, 0))
    return out


def run_decode(workload: str, cta: int = 0):
    """Runs fa_decode on the decode workload through the debug build with the
    partials kernel stamping its events (the balanced kernel's, for the
    shapes it takes). Returns (stamps, key tiles of the traced CTA)."""
    import torch

    from . import attention as fa
    from . import _abi
    from .workloads import DECODE_WORKLOADS, make_decode_inputs

    w = DECODE_WORKLOADS[workload]
    inp = make_decode_inputs(w)
    dev = torch.device("cuda", 0)
    L = w.lengths()
    q = inp.q.to(dev)
    kc = inp.k_cache.to(dev)
    vc = inp.v_cache.to(dev)
    lens = inp.cache_seqlens.to(dev)
    tb = None if inp.block_table is None else inp.block_table.to(dev)
    args = dict(q_len=w.q_len, max_seqlen_k=max(L), block_table=tb, page_size=inp.page_size,
                causal=w.causal)
    buf = torch.zeros(_abi.DEBUG_TRACE_BYTES // 8, dtype=torch.int64, device=dev)
    with fa.debug_build() as lib:
        assert lib.fa_debug_build() == 1
        fa.decode(q, kc, vc, lens, **args)   # warm-up
        _abi.check(lib.fa_debug_set_trace(buf.data_ptr(), buf.numel() * 8, cta), "trace")
        fa.decode(q, kc, vc, lens, **args)
        _abi.check(lib.fa_debug_set_trace(None, 0, 0), "trace")
        st, where = fa.check_device_error(dev)
        if st != 0:
            raise RuntimeError(f"device error {st} at {where:#x}")
    stamps = buf.view(32, 1024).cpu().numpy()
    return stamps, int((stamps[DEC_KINDS["M_PV"]] != 0).sum())


def run(kernel: str, workload: str, cta: int = 0):
    """Runs the forward (and, for ``bwd``, the backward) of the workload on
    cuda:0 through the debug build with stamping on for the kernel asked
    for. Returns (stamps [32, 1024] int64 numpy, steps of the traced CTA)."""
    import torch

    from . import attention as fa
    from . import _abi
    from .workloads import WORKLOADS, make_inputs

    if kernel == "dec":
        return run_decode(workload, cta)
    if kernel == "d64" and WORKLOADS[workload].D != 64:
        raise ValueError("--kernel d64 takes a D = 64 workload")

    w = WORKLOADS[workload]
    inp = make_inputs(w)
    B = len(inp.cu_seqlens) - 1
    dev = torch.device("cuda", 0)

    def to_dev(t):
        t = t.to(dev)
        return t if inp.varlen else t.view(B, w.N, t.shape[1], w.D)

    q, k, v, do = (to_dev(t) for t in (inp.q, inp.k, inp.v, inp.do))
    kw = dict(causal=w.causal, scale=w.scale)
    if inp.varlen:
        kw.update(cu_seqlens=inp.cu_seqlens.to(dev), max_seqlen=inp.max_seqlen)
    buf = torch.zeros(_abi.DEBUG_TRACE_BYTES // 8, dtype=torch.int64, device=dev)
    with fa.debug_build() as lib:
        assert lib.fa_debug_build() == 1
        if kernel in ("fwd", "d64"):
            _abi.check(lib.fa_debug_set_trace(buf.data_ptr(), buf.numel() * 8, cta), "trace")
            o, lse = fa.fwd(q, k, v, **kw)
            _abi.check(lib.fa_debug_set_trace(None, 0, 0), "trace")
        else:
            o, lse = fa.fwd(q, k, v, **kw)
            T = q.numel() // (w.H * w.D)
            ws = torch.empty(fa.workspace_size(T, w.H, w.D, q.dtype), dtype=torch.uint8,
                             device=dev)
            fa.bwd(do, q, k, v, o, lse, workspace=ws, phases=_abi.BWD_PREPROCESS, **kw)
            _abi.check(lib.fa_debug_set_trace(buf.data_ptr(), buf.numel() * 8, cta), "trace")
            fa.bwd(do, q, k, v, o, lse, workspace=ws, phases=_abi.BWD_FUSED_KERNEL, **kw)
            _abi.check(lib.fa_debug_set_trace(None, 0, 0), "trace")
            fa.bwd(do, q, k, v, o, lse, workspace=ws, phases=_abi.BWD_DQ_CONVERT, **kw)
        st, where = fa.check_device_error(dev)
        if st != 0:
            raise RuntimeError(f"device error {st} at {where:#x}")
    stamps = buf.view(32, 1024).cpu().numpy()
    # Steps of the traced CTA: query steps (backward) or key tiles (forward;
    # the second query tile of a causal pair has one more than the first).
    firsts = {"bwd": ["S_SFULL"], "fwd": ["W0_SFULL", "W1_SFULL"], "d64": ["W_SFULL"]}[kernel]
    kinds = {"bwd": BWD_KINDS, "fwd": FWD_KINDS, "d64": D64_KINDS}[kernel]
    n = max(int((stamps[kinds[f]] != 0).sum()) for f in firsts)
    return stamps, n


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--kernel", choices=["fwd", "bwd", "dec", "d64"], required=True)
    ap.add_argument("--workload", default="bf16_causal_b2_h16_n8192_d128")
    ap.add_argument("--cta", type=int, default=0)
    args = ap.parse_args(argv)
    from .build import build
    build(debug=True)
    stamps, n = run(args.kernel, args.workload, args.cta)
    kinds, table = {"bwd": (BWD_KINDS, BWD_SPANS), "fwd": (FWD_KINDS, FWD_SPANS),
                    "dec": (DEC_KINDS, DEC_SPANS), "d64": (D64_KINDS, D64_SPANS)}[args.kernel]
    print(f"{args.kernel} {args.workload} CTA {args.cta}: {n} steps stamped; cycles over "
          f"the steady-state steps")
    if args.kernel in ("dec", "d64"):
        for line in cta_report(stamps):
            print(line)
        stamps = stamps.copy()
        stamps[CTA_SM:CTA_END + 1] = 0
    nz = stamps[stamps != 0]
    if nz.size:
        span = int(nz.max()) - int(nz.min())
        print(f"  first to last stamp: {span} cycles, {span / max(n, 1):.0f} per step")
    print(f"  {'':62s} {'median':>8s} {'mean':>8s} {'p90':>8s}")
    for label, med, mean, p90, cnt in spans(stamps, kinds, table, n):
        if med is None:
            print(f"  {label:62s} {'-':>8s}  (0)")
        else:
            print(f"  {label:62s} {med:8.0f} {mean:8.0f} {p90:8.0f}  ({cnt})")
    return 0


if __name__ == "__main__":
    sys.exit(main())
