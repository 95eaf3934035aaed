"""Where the fused score kernel's time goes, per warp role.

    python -m streaming_top_lightning_b200.role_clocks [--workload v4flash_s16k]
        [--topk K] [--key-chunk C] [--steps N]

Builds and loads the profiling variant of the library (libstreamindex_roles.so,
the same sources compiled with SI_ROLE_CLOCKS), runs the indexer step on the
seeded synthetic inputs of a workload, and prints, per role, the cycles each
CTA spends in total, waiting on each barrier and in each selection phase
(mean over CTAs and steps, and as a share of the MMA warp's lifetime, which
spans the kernel), plus event counts.  The counters cost a few percent of
time, so the kernel time printed here is not a benchmark number.
"""

from __future__ import annotations

import argparse
import os
import sys

import numpy as np

ROLE_SLOTS = 32
NAMES = [
    ("producer: total", "c"), ("producer: wait key-tile stage free", "c"),
    ("producer: wait query tile free", "c"), ("producer: wait unit ring slot", "c"),
    ("MMA: total", "c"), ("MMA: wait key tile loaded", "c"),
    ("MMA: wait accumulator free", "c"), ("MMA: wait query tile loaded", "c"),
    ("MMA: wait unit", "c"),
    ("epilogue: total (sum over warps)", "c"), ("epilogue: wait unit", "c"),
    ("epilogue: wait strip free", "c"), ("epilogue: wait accumulator full", "c"),
    ("selection: total (sum over warps)", "c"), ("selection: wait strip full", "c"),
    ("selection: strip intake", "c"), ("selection: unit end (trim/merge, emit)", "c"),
    ("selection: prune/select inside intake", "c"),
    ("selection: prunes", "n"), ("selection: radix selects", "n"),
    ("selection: keys appended", "n"), ("selection: strips taken", "n"),
    ("selection: wait for partner at unit end", "c"),
    ("units", "n"), ("key tiles", "n"), ("selection: visible keys taken", "n"),
]


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="v4flash_s16k")
    ap.add_argument("--topk", type=int, default=0)
    ap.add_argument("--key-chunk", type=int, default=0)
    ap.add_argument("--steps", type=int, default=5)
    args = ap.parse_args(argv)

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    if root not in sys.path:
        sys.path.insert(0, root)
    import torch

    import synth
    from streaming_top_lightning_b200 import _lib, build

    lib = _lib.load(build.build(roles=True))
    import streaming_top_lightning_b200 as stl

    sh = synth.shape(args.workload, **({"topk": args.topk} if args.topk else {}))
    q = synth.gen_q(sh, 0, threads=16)
    qd = torch.from_numpy(q.view(np.int16)).cuda().view(torch.bfloat16)
    del q
    wd = torch.from_numpy(synth.gen_w(sh, 0)).cuda()
    kd = torch.from_numpy(synth.gen_kc(sh, 0).view(np.int16)).cuda().view(torch.bfloat16)
    plan = stl.plan(sh.B, sh.S, sh.H, sh.D, sh.m, sh.topk,
                    opts=stl.options(key_chunk=args.key_chunk))
    nblk = plan["query_blocks"]
    out = (torch.empty((sh.B, sh.S, sh.topk), dtype=torch.int32, device="cuda"),
           torch.empty((sh.B, sh.S, sh.topk), dtype=torch.float32, device="cuda"))
    for _ in range(2):
        stl.indexer_topk(qd, wd, kd, sh.m, sh.topk, out=out,
                         opts=stl.options(key_chunk=args.key_chunk))
    buf = np.zeros(1024 * ROLE_SLOTS, dtype=np.uint64)
    _lib.check("si_role_cycles", lib.si_role_cycles(buf.ctypes.data, buf.size, 1))
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nblk)]
           for _ in range(args.steps)]
    for lst in evs:
        for e in lst:
            e.record()
    torch.cuda.synchronize()
    for lst in evs:
        stl.indexer_topk(qd, wd, kd, sh.m, sh.topk, out=out,
                         opts=stl.options(key_chunk=args.key_chunk, score_event_list=lst))
    torch.cuda.synchronize()
    assert stl.device_error() == 0
    ms = np.mean([sum(lst[2 * b].elapsed_time(lst[2 * b + 1]) for b in range(nblk))
                  for lst in evs])
    _lib.check("si_role_cycles", lib.si_role_cycles(buf.ctypes.data, buf.size, 1))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    epi_warps, sel_warps = 8, 4  # warps per CTA of the two summed roles
    a = buf.reshape(1024, ROLE_SLOTS)[:sms].astype(np.float64) / args.steps
    life = a[:, 4].mean()
    print(f"{sh.name}: B={sh.B} S={sh.S} T={sh.T} H_I={sh.H} d_I={sh.D} top-{sh.topk} "
          f"key_chunk={args.key_chunk or 'one'}; plan {plan}")
    print(f"score kernel {ms:.3f} ms per step (profiling build); MMA-warp lifetime "
          f"{life / 1e6:.3f} Mcycles per CTA")
    print(f"{'role counter':44s} {'mean/CTA':>12s} {'max/CTA':>12s} {'share':>7s}"
          "  (share: per warp of the role, of the MMA-warp lifetime)")
    for i, (name, kind) in enumerate(NAMES):
        v = a[:, i]
        warps = epi_warps if name.startswith("epilogue") else (
            sel_warps if name.startswith("selection") else 1)
        if kind == "c":
            print(f"{name:44s} {v.mean() / 1e6:10.3f} M {v.max() / 1e6:10.3f} M "
                  f"{100 * v.mean() / warps / max(life, 1):6.1f}%")
        else:
            print(f"{name:44s} {v.mean():12.0f} {v.max():12.0f}")
    keys = a[:, 25].sum()
    if keys:
        print(f"selection intake: {a[:, 15].sum() / keys:.2f} cycles per visible key per warp; "
              f"{a[:, 20].sum() / keys:.3f} keys appended per key")
    return 0


if __name__ == "__main__":
    sys.exit(main())
