"""Run a number of fused loss calls on one synthetic workload, for profilers (ncu's
launch list or a single-kernel capture):

    python -m speculative_decoding_draft_vocab_b200.profile_call WORKLOAD [CALLS]

Exits with the device status of the last call (0 when no device-side flag was raised).
"""

import sys

import torch

from . import torch_api
from .synthetic import CONFIGS, make_inputs


def main(argv=None) -> int:
    argv = sys.argv[1:] if argv is None else argv
    name = argv[0] if argv else "recipe"
    calls = int(argv[1]) if len(argv) > 1 else 5
    if name not in CONFIGS:
        raise SystemExit(f"unknown workload {name!r}; one of {sorted(CONFIGS)}")
    inp = make_inputs(name, device="cuda")
    call = torch_api.Call(inp, rows=False)
    for _ in range(calls):
        call.launch()
    torch.cuda.synchronize()
    status = call.check_status()
    print(name, "status", status, "supervised rows", int(call.out.num_tokens.item()))
    return status


if __name__ == "__main__":
    sys.exit(main())
