"""Host-resident batches streamed through the device in groups of heads.

The (batch, head) units of the ELSAA operator are independent, and a
[B, H, N, d] tensor holds them one after another, so a step over a batch that
lives in pinned host memory can run as a pipeline over groups of units on
three CUDA streams: the copy-in of group g + 1, the forward and backward of
group g (libelsaa calls on the group's slice) and the copy-out of group g - 1
overlap.  Two device slots alternate between groups.  The shared gate and
lambda gradients are sums over every unit: each group's partial sums are
copied out with its gradients and added on the host in group order.

Plumbing only: the device work is the library's kernels and the copies; no
other device computation runs.
"""

from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as B


class HostStepPipeline:
    """Forward + backward of ELSAA over host-resident batches.

    params: the whole batch's elsaa_params (B, H, N, d, ...).  groups: how many
    groups of units the batch is split into (must divide B * H).  Inputs and
    outputs of step() are pinned host tensors of shape [B, H, N, d]."""

    def __init__(self, params: B.Params, groups: int, device, r_sort, r_race, gate_w, gate_b,
                 lam):
        BH = params.B * params.H
        if groups < 1 or BH % groups:
            raise ValueError(f"groups ({groups}) must divide B * H ({BH})")
        self.p = params
        self.groups = groups
        self.per = BH // groups
        self.dev = torch.device(device)
        # one group's problem: the same operator on `per` units
        self.pg = B.Params.make(1, self.per, params.N, params.d, params.torch_dtype,
                                params.sort_bits, params.chunk, params.race_tables,
                                params.race_bits, params.scale, params.gate_fixed,
                                params.gate_s, params.gate_r,
                                {v: k for k, v in B.SORT_ORDERS.items()}[params.sort_order],
                                params.lookback, params.causal, params.hash_rounds)
        self.small = {"r_sort": r_sort.to(self.dev), "r_race": r_race.to(self.dev),
                      "gate_w": gate_w.to(self.dev), "gate_b": gate_b.to(self.dev),
                      "lam": lam.to(self.dev)}
        dt, N, d = params.torch_dtype, params.N, params.d
        shape = (1, self.per, N, d)
        self.slots = []
        for _ in range(2):
            self.slots.append({
                "in": {k: torch.empty(shape, dtype=dt, device=self.dev) for k in
                       ("q", "k", "v", "dy")},
                "out": {k: torch.empty(shape, dtype=dt, device=self.dev) for k in
                        ("y", "dq", "dk", "dv")},
                "pg": [torch.empty(2, d, dtype=torch.float32, device=self.dev),
                       torch.empty(2, dtype=torch.float32, device=self.dev),
                       torch.empty(1, dtype=torch.float32, device=self.dev)],
                "saved": B.alloc_saved(self.pg, self.dev),
                "ws": B.alloc_workspace(self.pg, self.dev),
                "ev_in": torch.cuda.Event(), "ev_comp": torch.cuda.Event(),
                "ev_out": torch.cuda.Event(),
            })
        # every group's parameter-gradient partial sums, copied out
        self.pg_host = torch.empty(groups, 2 * d + 3, dtype=torch.float32, pin_memory=True)
        self.s_in = torch.cuda.Stream(self.dev)
        self.s_comp = torch.cuda.Stream(self.dev)
        self.s_out = torch.cuda.Stream(self.dev)
        self.n = 0   # groups enqueued so far (the slot use count runs across steps)

    def h2d_bytes(self, host: Dict[str, torch.Tensor]) -> int:
        return sum(host[k].numel() * host[k].element_size() for k in ("q", "k", "v", "dy"))

    def enqueue(self, host: Dict[str, torch.Tensor], out: Dict[str, torch.Tensor],
                stream: Optional[torch.cuda.Stream] = None) -> None:
        """Enqueue one step: host["q"|"k"|"v"|"dy"] in, out["y"|"dq"|"dk"|"dv"]
        written, all pinned [B, H, N, d]; the groups' parameter-gradient partial
        sums land in self.pg_host.  The step starts after the work already on
        `stream` (default: current), and `stream` waits for the whole step; call
        gradients() after synchronising it."""
        self.start_after(stream)
        self.enqueue_chained(host, out)
        self.join(stream)

    def start_after(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """What is enqueued next starts after the work already on `stream`
        (default: current)."""
        main = stream if stream is not None else torch.cuda.current_stream(self.dev)
        start = torch.cuda.Event()
        start.record(main)
        for s in (self.s_in, self.s_comp, self.s_out):
            s.wait_event(start)

    def enqueue_chained(self, host: Dict[str, torch.Tensor], out: Dict[str, torch.Tensor]) -> None:
        """Enqueue one step behind the steps enqueued before it on the
        pipeline's own streams, without waiting for any other stream: the
        first groups' copy-in overlaps the previous step's last compute and
        copy-out.  For back-to-back steps over host data; join() makes a
        stream wait for everything enqueued so far.  (out and pg_host are
        rewritten by every step.)"""
        BH, N, d = self.groups * self.per, self.p.N, self.p.d
        hin = {k: host[k].view(BH, N, d) for k in ("q", "k", "v", "dy")}
        hout = {k: out[k].view(BH, N, d) for k in ("y", "dq", "dk", "dv")}
        sm = self.small
        for g in range(self.groups):
            n = self.n
            self.n += 1
            sl = self.slots[n % 2]
            u0, u1 = g * self.per, (g + 1) * self.per
            with torch.cuda.stream(self.s_in):
                if n >= 2:
                    self.s_in.wait_event(sl["ev_comp"])   # the slot's inputs are free again
                for k in hin:
                    sl["in"][k][0].copy_(hin[k][u0:u1], non_blocking=True)
                sl["ev_in"].record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(sl["ev_in"])
                if n >= 2:
                    self.s_comp.wait_event(sl["ev_out"])   # the slot's outputs are out
                i, o = sl["in"], sl["out"]
                B.forward(self.pg, i["q"], i["k"], i["v"], sm["r_sort"], sm["r_race"],
                          sm["gate_w"], sm["gate_b"], sm["lam"], y=o["y"], saved=sl["saved"],
                          ws=sl["ws"], stream=self.s_comp)
                B.backward(self.pg, i["q"], i["k"], i["v"], sm["r_sort"], sm["r_race"],
                           sm["gate_w"], sm["gate_b"], sm["lam"], sl["saved"], i["dy"], o["dq"],
                           o["dk"], o["dv"], *sl["pg"], ws=sl["ws"], stream=self.s_comp)
                sl["ev_comp"].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(sl["ev_comp"])
                for k in hout:
                    hout[k][u0:u1].copy_(sl["out"][k][0], non_blocking=True)
                row = self.pg_host[g]
                row[:2 * d].copy_(sl["pg"][0].view(-1), non_blocking=True)
                row[2 * d:2 * d + 2].copy_(sl["pg"][1], non_blocking=True)
                row[2 * d + 2:].copy_(sl["pg"][2], non_blocking=True)
                sl["ev_out"].record(self.s_out)

    def join(self, stream: Optional[torch.cuda.Stream] = None) -> None:
        """`stream` (default: current) waits for every step enqueued so far."""
        main = stream if stream is not None else torch.cuda.current_stream(self.dev)
        for s in (self.s_in, self.s_comp, self.s_out):
            main.wait_stream(s)

    def gradients(self):
        """(dgate_w [2, d], dgate_b [2], dlambda [1]) of the last step, summed
        over the groups in group order on the host (fp64 sums)."""
        d = self.p.d
        tot = self.pg_host.double().sum(0)
        return (tot[:2 * d].view(2, d).float(), tot[2 * d:2 * d + 2].float(),
                tot[2 * d + 2:].float())
