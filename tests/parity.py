"""Helpers that compare the CUDA path (through the C ABI) with the CPU oracle.

Gates (the block's accuracy contract):
  * expert ids: on every token whose selection margin exceeds TIE_MARGIN the
    sorted id set equals the oracle's (near-ties are counted, not gated);
  * gating weights: relative error <= 1e-5 on those tokens;
  * output: |gpu - ref| <= 2e-2 * (1 + |ref|) elementwise, where ref is the
    float64 oracle evaluated with the GPU's expert choice (so near-tie tokens
    are compared too).
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from routed_moe_layer_b200.ops import BlockConfig

TIE_MARGIN = 1e-4
OUT_RTOL = 2e-2
W_RTOL = 1e-5


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def oracle_cfg(cfg: BlockConfig) -> oracle.MoeConfig:
    return oracle.MoeConfig(E=cfg.E, I=cfg.I, I_shared=cfg.I_shared, top_k=cfg.top_k,
                            n_group=cfg.n_group, topk_group=cfg.topk_group,
                            routed_scaling_factor=cfg.routed_scaling_factor,
                            norm_topk_prob=cfg.norm_topk_prob)


def np_inputs(d: dict) -> dict:
    return {k: (None if v is None else to_np(v)) for k, v in d.items()}


def check_routing(ids_gpu: torch.Tensor, w_gpu: torch.Tensor, xn, Wrn, biasn, cfg: BlockConfig,
                  rows=None, token_mask=None):
    """Gate the GPU routing against the oracle; returns a small report.  With a
    token mask, padding tokens must have ids -1 and weights 0 exactly."""
    ocfg = oracle_cfg(cfg)
    if rows is not None:
        xn = xn[rows]
    ids_ref, w_ref, margin, _ = oracle.route(xn, Wrn, biasn, ocfg)
    ig = ids_gpu.cpu().numpy()
    wg = w_gpu.cpu().numpy().astype(np.float64)
    if rows is not None:
        ig, wg = ig[rows], wg[rows]
    if token_mask is not None:
        pad = np.asarray(token_mask).reshape(-1) == 0
        assert np.all(ig[pad] == -1) and np.all(wg[pad] == 0.0)
        ig, wg, ids_ref, w_ref, margin = ig[~pad], wg[~pad], ids_ref[~pad], w_ref[~pad], margin[~pad]
    far = margin > TIE_MARGIN
    og = np.argsort(ig, axis=1)
    orf = np.argsort(ids_ref, axis=1)
    ig_s = np.take_along_axis(ig, og, 1)
    ir_s = np.take_along_axis(ids_ref, orf, 1)
    mism = np.nonzero(far & np.any(ig_s != ir_s, axis=1))[0]
    assert mism.size == 0, f"{mism.size} tokens with margin > {TIE_MARGIN} route differently, e.g. {mism[:5]}"
    wg_s = np.take_along_axis(wg, og, 1)[far]
    wr_s = np.take_along_axis(w_ref, orf, 1)[far]
    rel = np.abs(wg_s - wr_s) / np.abs(wr_s)
    assert rel.size == 0 or rel.max() <= W_RTOL, f"weight rel err {rel.max():.3g}"
    # ids valid, distinct per token, ordered by descending c like the oracle
    assert ig.min() >= 0 and ig.max() < cfg.E
    assert np.all(np.sort(ig, axis=1)[:, 1:] != np.sort(ig, axis=1)[:, :-1])
    return dict(tokens=int(len(ig)), near_ties=int((~far).sum()),
                max_w_rel=float(rel.max()) if rel.size else 0.0)


def check_output(out_gpu: torch.Tensor, ids_gpu: torch.Tensor, d_np: dict, cfg: BlockConfig,
                 tokens=None, residual_np=None, token_mask=None):
    """Gate the GPU output against the float64 oracle under the GPU's expert
    choice, on all tokens or on the given token sample."""
    ocfg = oracle_cfg(cfg)
    ids = ids_gpu.cpu().numpy()
    args = (d_np["x"], d_np["Wr"], d_np["bias"], d_np["w13"], d_np["w2"],
            d_np.get("ws13"), d_np.get("ws2"), ocfg)
    if tokens is None:
        ref, _, _, _ = oracle.moe_forward(*args, residual=residual_np, ids=ids,
                                          token_mask=token_mask)
        got = to_np(out_gpu).astype(np.float64)
    else:
        tokens = np.asarray(tokens)
        ref, _, _, _ = oracle.moe_forward_tokens(tokens, *args, residual=residual_np, ids=ids,
                                                 token_mask=token_mask)
        got = to_np(out_gpu[torch.as_tensor(tokens, device=out_gpu.device)]).astype(np.float64)
    err = np.abs(got - ref)
    bound = OUT_RTOL * (1.0 + np.abs(ref))
    bad = np.argwhere(err > bound)
    assert bad.size == 0, (f"{len(bad)} outputs out of tolerance; worst err {err.max():.4g} "
                           f"at {np.unravel_index(err.argmax(), err.shape)}")
    assert np.all(np.isfinite(got))
    return dict(max_abs_err=float(err.max()), max_ref=float(np.abs(ref).max()),
                rms_rel=float(np.sqrt(np.mean(err ** 2) / max(np.mean(ref ** 2), 1e-30))))
