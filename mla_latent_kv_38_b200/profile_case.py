"""Run a workload's decode step a fixed number of times, for profilers.

    python -m mla_latent_kv_38_b200.profile_case --workload v2_decode --iters 4 [--impl 0] [--cache e4m3]

Sets up the workload (cache history appended through the library), then runs
`--iters` full steps (absorb_q, rope_append, decode, up_v) back to back and
exits; nothing is timed here.
"""

import argparse

import torch

from .runner import DeviceCase
from .workloads import workload_specs


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="v2_decode")
    ap.add_argument("--iters", type=int, default=4)
    ap.add_argument("--impl", type=int, default=0)
    ap.add_argument("--decode-only", action="store_true")
    ap.add_argument("--cache", choices=["bf16", "e4m3"], default="bf16")
    a = ap.parse_args()
    dc = DeviceCase(workload_specs()[a.workload], impl=a.impl, cache=a.cache)
    for _ in range(a.iters):
        dc.reset_step_inputs()
        if a.decode_only:
            dc.decode_only()
        else:
            dc.step()
    torch.cuda.synchronize()
    st = dc.decode_status() | dc.append_status()
    if st:
        raise SystemExit(f"device status {st}")
    print("ok")


if __name__ == "__main__":
    main()
