"""Runs the routed-expert call of one synthetic MoE layer a few times, so that
a profiler can capture its kernels on a case that holds only one layer on the
device (the benchmark rotates many layers and token batches, too much device
memory for a multi-pass capture).

    python -m bit_expert_gemm_b200.profile_case --fmt bf16 --tokens 1 --calls 4
    ncu --set full --clock-control none -k regex:k_decode_ffn -s 3 -c 1 \\
        python -m bit_expert_gemm_b200.profile_case --fmt bf16 --tokens 1 --calls 4

The routing is drawn by the library's own router (moe_route_permute) from
the synthetic tokens and router weights, as in a layer forward; the expert
call is the one MoELayer makes for the format: moe_experts_bf16 (routed +
shared experts), moe_experts_awq_g32_prepacked (routed AWQ + FP16 shared
experts) or moe_grouped_swiglu_nvfp4_prepacked (routed NVFP4 experts).
With --layer the whole layer forward (MoELayer: routing, experts, shared
expert, combine) runs instead, for launch lists of a complete step.
"""

from __future__ import annotations

import argparse
import dataclasses

import torch

from . import abi, synth
from .layer import MoELayer, prepare_nvfp4_weights

WORKLOAD_OF = {"bf16": "bf16", "awq_g32": "awq_g32", "nvfp4": "nvfp4"}


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--fmt", choices=sorted(WORKLOAD_OF), default="bf16")
    ap.add_argument("--tokens", type=int, default=1)
    ap.add_argument("--experts", type=int, default=0, help="override E (0: the workload's)")
    ap.add_argument("--calls", type=int, default=4)
    ap.add_argument("--seed", type=int, default=1)
    ap.add_argument("--layer", action="store_true", help="the whole layer forward instead of the expert call")
    a = ap.parse_args(argv)
    if not torch.cuda.is_available():
        raise SystemExit("profile_case needs a CUDA device")
    wl = synth.WORKLOADS[WORKLOAD_OF[a.fmt]]
    if a.experts:
        wl = dataclasses.replace(wl, E=a.experts)
    dev = "cuda"
    w = synth.make_weights(wl, seed=a.seed, device=dev)
    x = synth.make_tokens(wl, a.tokens, seed=a.seed, device=dev)
    _, _, _, off, rt, _ = abi.moe_route_permute(x, w["w_router"], w["bias"], wl.k)
    rows = a.tokens * wl.k
    if a.layer:
        layer = MoELayer(w, wl.k, a.fmt, T_max=a.tokens)

        def call():
            layer.forward(x)
    elif a.fmt == "nvfp4":
        w = prepare_nvfp4_weights(w)
        for key in ("w_gate_up", "w_down"):
            del w[key]
        torch.cuda.empty_cache()
        xb = x if x.dtype == torch.bfloat16 else x.to(torch.bfloat16)

        def call():
            abi.moe_grouped_swiglu_nvfp4_prepacked(xb, rt, off, rows, w["w_gu"], w["sfp_gu"], w["gs_gu"], w["w_d"],
                                                   w["sfp_d"], w["gs_d"])
    elif a.fmt == "awq_g32":
        # as MoELayer does: the expert call reads the tile-packed copy of the routed weights
        packed = abi.moe_awq_prepack_g32(w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"], w["qz_d"], w["sc_d"])

        def call():
            abi.moe_experts_awq_g32_prepacked(x, rt, off, rows, w["qw_gu"], w["qz_gu"], w["sc_gu"], w["qw_d"],
                                              w["qz_d"], w["sc_d"], packed, w["w_sh_gate_up"], w["w_sh_down"])
    else:
        def call():
            abi.moe_experts_bf16(x, rt, off, rows, w["w_gate_up"], w["w_down"], w["w_sh_gate_up"], w["w_sh_down"])
    for _ in range(a.calls):
        call()
    torch.cuda.synchronize()
    status = abi.moe_device_status()
    if status != 0:
        raise SystemExit(f"device status {status}")
    print(f"{a.fmt}: T={a.tokens} E={wl.E} rows={rows} calls={a.calls} "
          f"peak device memory {torch.cuda.max_memory_allocated() / 1e9:.2f} GB")


if __name__ == "__main__":
    main()
