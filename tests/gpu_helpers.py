"""Shared machinery of the GPU parity tests: draw a workload on the GPU,
run the CUDA path through the C ABI, and evaluate the oracle on the CPU from
the same generator bytes (weights quantised by the oracle itself)."""

from __future__ import annotations

import numpy as np
import torch

from moe_layer_top_b200 import inputs, ops
from oracle import moe_oracle as O

# output tolerances: normwise relative error and max |diff| / max |ref|
TOL_BF16 = 5e-3
TOL_FP8 = 2e-2
TOL_MAX_REL = 0.05


class LazyExperts:
    """Per-expert host copies of the generator's bf16 weights (bit patterns),
    and the oracle's own FP8 (block-128 or MX) quantisation of them, made on
    first access."""

    def __init__(self, w_dev: torch.Tensor, fp8: bool, mx: bool = False):
        self.w_dev = w_dev
        self.fp8 = fp8
        self.mx = mx
        self._cache = {}

    def _get(self, e):
        e = int(e)
        if e not in self._cache:
            w = self.w_dev[e].view(torch.int16).cpu().numpy().view(np.uint16)     # bf16 bit patterns
            if self.mx:
                self._cache[e] = O.quantize_mx_group32(w)
            else:
                self._cache[e] = O.quantize_weight_block128(w) if self.fp8 else (w, None)
        return self._cache[e]

    @property
    def codes(self):
        outer = self

        class _C:
            def __getitem__(self, e):
                return outer._get(e)[0]
        return _C()

    @property
    def scales(self):
        outer = self

        class _S:
            def __getitem__(self, e):
                return outer._get(e)[1]
        return _S()


class Case:
    """One workload instance on the GPU plus its oracle evaluation."""

    def __init__(self, cfg: inputs.MoEConfig, T: int, seed: int = 0, mode=ops.MODE_AUTO, block_m=0,
                 weights=None, split_k=True, router_weight_on_input=False, swiglu_limit=0.0, renormalize=True,
                 persistent_decode=False):
        self.cfg, self.T, self.seed = cfg, T, seed
        self.renormalize = renormalize
        self.router_weight_on_input, self.swiglu_limit = router_weight_on_input, swiglu_limit
        dev = torch.device("cuda")
        if weights is None:
            weights = inputs.make_weights(cfg, seed, device=dev)
        self.w13_bf16, self.w2_bf16 = weights
        self.x = inputs.make_tokens(cfg, T, seed, device=dev)
        self.routing = inputs.make_routing(cfg, T, seed, device=dev)
        if cfg.mx:
            self.w13, self.w13_scale = ops.quantize_weights_mxfp8(self.w13_bf16)
            self.w2, self.w2_scale = ops.quantize_weights_mxfp8(self.w2_bf16)
        elif cfg.fp8:
            self.w13, self.w13_scale = ops.quantize_weights_fp8(self.w13_bf16)
            self.w2, self.w2_scale = ops.quantize_weights_fp8(self.w2_bf16)
        else:
            self.w13, self.w2 = self.w13_bf16, self.w2_bf16
            self.w13_scale = self.w2_scale = None
        self.p = ops.problem(T, cfg.E, cfg.topk, cfg.H, cfg.I, fp8=cfg.fp8, mode=mode, block_m=block_m,
                             split_k=split_k, mx=cfg.mx, router_weight_on_input=router_weight_on_input,
                             swiglu_limit=swiglu_limit, renormalize=renormalize,
                             persistent_decode=persistent_decode)
        self.q = ops.resolve_problem(self.p)
        self.ws = ops.alloc_workspace(self.p)
        self.out = torch.empty((T, cfg.H), dtype=torch.bfloat16, device=dev)

    def run(self):
        ops.fused_forward(self.p, self.x, self.w13, self.w2, logits=self.routing.get("logits"),
                          topk_ids=self.routing.get("topk_ids"), topk_weights=self.routing.get("topk_weights"),
                          w13_scale=self.w13_scale, w2_scale=self.w2_scale, out=self.out, ws=self.ws)
        torch.cuda.synchronize()
        return self.out

    def views(self):
        return ops.workspace_views(self.p, self.ws)

    def status(self):
        return ops.read_status(self.p, self.ws)

    def _oracle_inputs(self):
        """Host copies of x and the routing input, and the oracle's lazily quantised experts
        (made once per case)."""
        if not hasattr(self, "_host"):
            kw = {}
            if "logits" in self.routing:
                kw["logits"] = self.routing["logits"].cpu().numpy()
            else:
                kw["topk_ids"] = self.routing["topk_ids"].cpu().numpy()
                kw["topk_weights"] = self.routing["topk_weights"].cpu().numpy()
            kw["router_weight_on_input"] = self.router_weight_on_input
            kw["renormalize"] = self.renormalize
            kw["swiglu_limit"] = self.swiglu_limit if self.swiglu_limit > 0 else None
            l13 = LazyExperts(self.w13_bf16, self.cfg.fp8, self.cfg.mx)
            l2 = LazyExperts(self.w2_bf16, self.cfg.fp8, self.cfg.mx)
            if self.cfg.fp8:
                kw.update(w13_scale=l13.scales, w2_scale=l2.scales, mx=self.cfg.mx)
            self._host = (self.x.float().cpu().double().numpy(), l13.codes, l2.codes, kw)
        return self._host

    def oracle(self, tokens=None, return_y=False):
        x, w13, w2, kw = self._oracle_inputs()
        return O.moe_forward(x, w13, w2, self.cfg.topk, tokens=tokens, return_y=return_y, **kw)

    def oracle_assignments(self, flat):
        """The oracle's unweighted expert outputs of the flat assignments t * topk + j."""
        x, w13, w2, kw = self._oracle_inputs()
        return O.assignment_outputs(x, w13, w2, self.cfg.topk, flat, **kw)


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    diff = got - ref
    norm_rel = np.linalg.norm(diff) / max(np.linalg.norm(ref), 1e-30)
    max_rel = np.abs(diff).max() / max(np.abs(ref).max(), 1e-30)
    return float(norm_rel), float(max_rel)


def assert_close(got, ref, fp8: bool):
    nr, mr = errors(got, ref)
    tol = TOL_FP8 if fp8 else TOL_BF16
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), "non-finite output"
    assert nr <= tol, f"normwise relative error {nr:.3e} > {tol}"
    assert mr <= TOL_MAX_REL, f"max |diff| / max |ref| = {mr:.3e} > {TOL_MAX_REL}"
    return nr, mr
