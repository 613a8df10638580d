"""Plain CPU oracle of the LingBot-Video / DeepSeek-V3-style routed MoE block.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the product path.

Sources (web pages; cited by title and section):

[S1] prhub report "sglang PR #32341: LingBot-Video MoE 30B text-to-video".
     Section "实现拆解" (implementation breakdown), step 1: the router computes
     in fp32 with sigmoid scoring plus ``e_score_correction_bias`` and a
     group-limited top-k; the router pre-scales the top-k scores, so the
     expert kernel must not scale a second time.  Section "关键源码片段"
     (key source snippets), ``LingBotVideoSparseMoeBlock``: the routing record
     is fp32 weights + int32 ids; experts run SiLU-gated with the router
     weight applied on the output (``apply_router_weight_on_input=False``);
     ``w13`` is packed [E, 2I, H] non-interleaved (gate rows, then up rows);
     the shared expert is added unscaled.  Section "风险与影响" (risks),
     item 4: group score is the sum of the top-2 scores inside a group, and
     the number of experts must be divisible by ``n_group``.
[S2] xxqk.cn article "vLLM-Omni 原生推理 LingBot-Video", section
     "MoE 实现的源码级要点" (source-level MoE notes): selection uses the
     bias-corrected scores while the gating weights use the raw scores;
     ``norm_topk_prob`` renormalisation; tokens reordered by expert, expert
     GEMMs in bf16, restored by an fp32 scatter-weighted sum; a shared expert
     is added when ``n_shared_experts > 0``; RMSNorm accumulates in fp32.
[S3] vLLM-Omni recipe "Robbyant/LingBot-Video.md", section on MoE
     validation: router weights and correction bias are kept in fp32, routed
     and shared expert weights are bf16.

Precision.  The pages fix the router to fp32, so the router scores that
decide the integer expert choice are fp32 values here too: each logit is
the exact (float64) dot product rounded once to fp32, the sigmoid is
evaluated in float64 and rounded once to fp32, and the bias is added in
fp32.  Everything downstream of the choice (weights, expert MLPs, restore,
shared expert, residual) is float64 on the bf16 input values: the exact
result that a bf16/fp32 implementation approximates.

Readings where the pages are silent (each is also listed in the design
notes of the repository):
  * ties in every selection go to the higher value, then the lower index
    (a stable descending sort);
  * experts outside the kept groups are excluded (score -inf), not zeroed;
  * group scores use the bias-corrected scores c, like the expert choice;
  * ``norm_topk_prob`` is on; the denominator has no epsilon guard;
  * ids are returned in selection order (descending c);
  * the padding mask is per token: a padding token takes no routed expert
    (id -1, weight 0) and keeps the shared expert (see ``apply_token_mask``);
  * FP8 expert weights are E4M3 codes with one power-of-two scale per
    128 x 128 block (see ``fp8_block_dequant``).
"""

from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    """Block hyper-parameters ([S1] "实现拆解" step 3: 128 experts, top-8,
    moe_intermediate_size=768, n_group=4, topk_group=2, scaling 2.5)."""

    E: int = 128
    I: int = 768
    I_shared: int = 768
    top_k: int = 8
    n_group: int = 4
    topk_group: int = 2
    routed_scaling_factor: float = 2.5
    norm_topk_prob: bool = True


# ----------------------------------------------------------------------------
# bf16 rounding (round-to-nearest-even), used only where the method itself
# casts to bf16: the MoE input of a stacked layer (RMSNorm output).
# ----------------------------------------------------------------------------
def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round finite values to the nearest bf16 (ties to even); returns float32."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32)


# ----------------------------------------------------------------------------
# Router ([S1] "实现拆解" step 1; [S2] "Router 的不对称选路")
# ----------------------------------------------------------------------------
def router_scores(x: np.ndarray, Wr: np.ndarray, bias: np.ndarray):
    """fp32 router scores.

    x [T,H] (bf16 values), Wr [E,H] fp32, bias [E] fp32.
    Returns (logits, s, c), all fp32 [T,E]:
      logits = x . Wr^T   (exact dot product, rounded once to fp32)
      s      = sigmoid(logits)              (raw scores: gating weights)
      c      = s + bias                     (bias-corrected: selection only)
    """
    logits = (x.astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    s = (1.0 / (1.0 + np.exp(-logits.astype(np.float64)))).astype(np.float32)
    c = s + bias.astype(np.float32)[None, :]  # fp32 + fp32 -> fp32
    return logits, s, c.astype(np.float32)


def group_limited_topk(c: np.ndarray, n_group: int, topk_group: int, top_k: int):
    """Group-limited top-k on bias-corrected scores c [T,E] (fp32).

    1. group score G_j = sum of the two largest c inside group j
       ([S1] "风险与影响" item 4), the sum taken in fp32;
    2. keep the ``topk_group`` groups with the largest G;
    3. choose the ``top_k`` largest c among the experts of the kept groups.

    Returns (ids [T,top_k] int32 in selection order, margin [T] float64) where
    margin = min(G_(g) - G_(g+1), c_(k) - c_(k+1) over the candidates): the
    distance of each token from a different choice (inf when no alternative).
    """
    T, E = c.shape
    if E % n_group != 0:
        raise ValueError("number of experts must be divisible by n_group")
    gs = E // n_group
    if not 1 <= topk_group <= n_group:
        raise ValueError("topk_group must lie in [1, n_group]")
    if topk_group * gs < top_k:
        raise ValueError("kept groups hold fewer experts than top_k")
    if topk_group < n_group:
        if gs < 2:
            raise ValueError("group-limited top-k needs at least 2 experts per group")
        cg = c.reshape(T, n_group, gs)
        # step 1: top-2 inside each group (stable descending order, lower index first)
        order_in_group = np.argsort(-cg, axis=2, kind="stable")
        top2 = np.take_along_axis(cg, order_in_group[:, :, :2], axis=2)
        G = (top2[:, :, 0] + top2[:, :, 1]).astype(np.float32)  # [T, n_group]
        # step 2: keep the best topk_group groups
        g_order = np.argsort(-G, axis=1, kind="stable")
        kept = g_order[:, :topk_group]
        keep_mask = np.zeros((T, n_group), dtype=bool)
        np.put_along_axis(keep_mask, kept, True, axis=1)
        expert_mask = np.repeat(keep_mask, gs, axis=1)  # [T, E]
    else:
        # every group is kept: the group step selects nothing
        expert_mask = np.ones((T, E), dtype=bool)
    # step 3: top_k over the candidate experts (others excluded with -inf)
    cand = np.where(expert_mask, c.astype(np.float64), -np.inf)
    e_order = np.argsort(-cand, axis=1, kind="stable")
    ids = e_order[:, :top_k].astype(np.int32)
    # distance from a different choice
    margin = np.full(T, np.inf)
    if topk_group < n_group:
        Gs = np.take_along_axis(G.astype(np.float64), g_order, axis=1)
        margin = np.minimum(margin, Gs[:, topk_group - 1] - Gs[:, topk_group])
    if topk_group * gs > top_k:
        cs = np.take_along_axis(cand, e_order, axis=1)
        margin = np.minimum(margin, cs[:, top_k - 1] - cs[:, top_k])
    return ids, margin


def routing_weights(s: np.ndarray, ids: np.ndarray, routed_scaling_factor: float,
                    norm_topk_prob: bool = True) -> np.ndarray:
    """Gating weights from the RAW scores s ([S2]: weights use the raw scores),
    renormalised over the chosen experts and scaled once by the routed scaling
    factor ([S1] step 1: the router pre-scales; the expert kernel does not).
    Returns float64 [T, top_k]."""
    sel = np.take_along_axis(s.astype(np.float64), ids.astype(np.int64), axis=1)
    if norm_topk_prob:
        sel = sel / sel.sum(axis=1, keepdims=True)
    return routed_scaling_factor * sel


def apply_token_mask(ids: np.ndarray, w: np.ndarray, margin: np.ndarray, token_mask):
    """Padding mask ([S2] "MoE 实现的源码级要点": in the forward the padding mask
    acts on the routing scores, which are then renormalised).

    Reading: the mask is per token (nonzero = real token, 0 = padding).  A
    padding token's routing scores are masked to zero, so it takes no routed
    expert: id -1 and weight 0 (renormalising an all-zero row keeps it zero).
    A real token's choice and weights are unchanged (its own scores are not
    masked, and renormalising them again is the identity).  The shared expert
    is dense and still applies to every token.
    Returns new (ids, w, margin); a padding token's margin is +inf (no choice).
    """
    real = np.asarray(token_mask).reshape(-1) != 0
    ids = np.array(ids, dtype=np.int32, copy=True)
    w = np.array(w, dtype=np.float64, copy=True)
    margin = np.array(margin, dtype=np.float64, copy=True)
    ids[~real] = -1
    w[~real] = 0.0
    margin[~real] = np.inf
    return ids, w, margin


def route(x, Wr, bias, cfg: MoeConfig, token_mask=None):
    """Full router: returns (ids int32 [T,k], w float64 [T,k], margin [T], s fp32 [T,E])."""
    _, s, c = router_scores(x, Wr, bias)
    ids, margin = group_limited_topk(c, cfg.n_group, cfg.topk_group, cfg.top_k)
    w = routing_weights(s, ids, cfg.routed_scaling_factor, cfg.norm_topk_prob)
    if token_mask is not None:
        ids, w, margin = apply_token_mask(ids, w, margin, token_mask)
    return ids, w, margin, s


# ----------------------------------------------------------------------------
# Token reorder ([S2] "_reorder_tokens": rows regrouped by expert before the
# grouped expert GEMMs).  Reading: rows ordered by expert, then token, which
# makes the permutation unique.
# ----------------------------------------------------------------------------
def permutation(ids: np.ndarray, E: int):
    """Returns (expert_offsets [E+1], row_of [T*k], tok_of [T*k]), int64.

    The (token, slot) entries flattened as t*k + j are sorted by expert with a
    stable sort (a token holds each expert at most once, so equal experts keep
    token order); row_of maps an entry to its row, tok_of a row to its token.
    """
    T, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")          # row -> flattened entry
    row_of = np.empty(T * k, dtype=np.int64)
    row_of[order] = np.arange(T * k)
    tok_of = order // k
    counts = np.bincount(flat, minlength=E)
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return offsets, row_of, tok_of


# ----------------------------------------------------------------------------
# Experts ([S1] "关键源码片段": activation silu, gated, non-interleaved w13)
# ----------------------------------------------------------------------------
def _silu(a: np.ndarray) -> np.ndarray:
    return a / (1.0 + np.exp(-a))


def swiglu_mlp(x: np.ndarray, w13: np.ndarray, w2: np.ndarray) -> np.ndarray:
    """One SwiGLU expert in float64.

    x [n,H]; w13 [2I,H] with gate rows 0..I-1 then up rows I..2I-1;
    w2 [H,I].  Returns (silu(x.Wg^T) * (x.Wu^T)) . W2^T as float64 [n,H].
    """
    I = w13.shape[0] // 2
    xd = x.astype(np.float64)
    gate = xd @ w13[:I].astype(np.float64).T
    up = xd @ w13[I:].astype(np.float64).T
    return (_silu(gate) * up) @ w2.astype(np.float64).T


def dense_ffn(x: np.ndarray, w13: np.ndarray, w2: np.ndarray, residual=None) -> np.ndarray:
    """Dense feed-forward layer ([S2] "MoE 实现的源码级要点": a block uses the sparse
    MoE block or a plain LingBotVideoMLP -- the dense FFN -- by decoder_sparse_step
    and layer index; the shared expert is the same MLP).  float64 [T,H]:
    out = SwiGLU(x; w13 [2I,H] gate|up, w2 [H,I]) (+ residual).  Pinned through
    ``swiglu_mlp``'s pins."""
    out = swiglu_mlp(x, w13, w2)
    if residual is not None:
        out = out + residual.astype(np.float64)
    return out


def moe_forward(x, Wr, bias, w13, w2, ws13, ws2, cfg: MoeConfig,
                residual=None, ids=None, token_mask=None):
    """Block output in float64 [T,H].

    out = sum_i w_i * Expert_{ids_i}(x)          (fp32 scatter-weighted restore, [S2])
        + SharedExpert(x)                        (added unscaled, [S1])
        + residual                               (only for a residual stack)

    ``ids`` may be given (e.g. to evaluate near-tie tokens under another
    implementation's choice); the weights are then recomputed from this
    oracle's own raw scores for those ids.  ``token_mask`` (per token,
    0 = padding) removes the routed part of padding tokens (``apply_token_mask``).
    Returns (out, ids, w, margin).
    """
    _, s, c = router_scores(x, Wr, bias)
    if ids is None:
        ids, margin = group_limited_topk(c, cfg.n_group, cfg.topk_group, cfg.top_k)
    else:
        ids = np.asarray(ids, dtype=np.int32)
        _, margin = group_limited_topk(c, cfg.n_group, cfg.topk_group, cfg.top_k)
    if token_mask is not None:
        ids = np.where((np.asarray(token_mask).reshape(-1) != 0)[:, None], ids, 0)
    w = routing_weights(s, ids, cfg.routed_scaling_factor, cfg.norm_topk_prob)
    if token_mask is not None:
        ids, w, margin = apply_token_mask(ids, w, margin, token_mask)
    T, H = x.shape
    out = np.zeros((T, H), dtype=np.float64)
    for e in range(w13.shape[0]):
        t_idx, slot = np.nonzero(ids == e)
        if t_idx.size == 0:
            continue
        y = swiglu_mlp(x[t_idx], w13[e], w2[e])
        np.add.at(out, t_idx, w[t_idx, slot][:, None] * y)
    if ws13 is not None and cfg.I_shared > 0:
        out += swiglu_mlp(x, ws13, ws2)
    if residual is not None:
        out += residual.astype(np.float64)
    return out, ids, w, margin


def moe_forward_tokens(tokens, x, Wr, bias, w13, w2, ws13, ws2, cfg: MoeConfig,
                       residual=None, ids=None, token_mask=None):
    """``moe_forward`` restricted to the token indices ``tokens`` (each token
    is computed in isolation, so this equals the corresponding rows of the
    full output).  Used to check full-size runs on a sample of outputs."""
    tokens = np.asarray(tokens, dtype=np.int64)
    res = None if residual is None else residual[tokens]
    sub_ids = None if ids is None else np.asarray(ids)[tokens]
    sub_mask = None if token_mask is None else np.asarray(token_mask).reshape(-1)[tokens]
    return moe_forward(x[tokens], Wr, bias, w13, w2, ws13, ws2, cfg,
                       residual=res, ids=sub_ids, token_mask=sub_mask)


# ----------------------------------------------------------------------------
# FP8 expert weights.  [S3] "Known limitations" names an optional FP8 backend
# of the upstream project and gives no format.  Reading: weight-only FP8 --
# every expert matrix (routed and shared) stored as OCP E4M3 codes ("fn"
# variant: no infinities) with one power-of-two scale per 128 x 128 block,
# held as a UE8M0 exponent byte; activations, router and restore unchanged.
# With power-of-two scales every dequantised weight is a bf16 value, so the
# FP8 block is exactly the bf16 block evaluated on the dequantised weights.
# ----------------------------------------------------------------------------
FP8_BLOCK = 128


def fp8_e4m3_decode(codes) -> np.ndarray:
    """E4M3 codes (uint8) to float64, from the format's definition: sign bit 7,
    exponent bits 6..3 (bias 7), mantissa bits 2..0.  Exponent 0 encodes
    zero and the subnormals m/8 * 2^-6; exponent 15 with mantissa 7 is NaN;
    every other code is (1 + m/8) * 2^(e-7) (largest: 448)."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = c >> 7
    e = (c >> 3) & 0xF
    m = c & 0x7
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where(sign == 1, -mag, mag)
    return np.where((e == 15) & (m == 7), np.nan, val)


def ue8m0_decode(exps) -> np.ndarray:
    """UE8M0 scale bytes to float64: 2^(s - 127); 255 is NaN."""
    s = np.asarray(exps, dtype=np.uint8).astype(np.float64)
    return np.where(s == 255, np.nan, np.exp2(s - 127.0))


def fp8_block_dequant(codes, scale_exp, block: int = FP8_BLOCK) -> np.ndarray:
    """Dequantised weights, float64 [..., N, K]: element (n, k) of each matrix
    is decode(codes[n, k]) * 2^(scale_exp[n // block, k // block] - 127).
    ``scale_exp`` is [..., ceil(N/block), ceil(K/block)] (a partial last
    block row / column has its own scale)."""
    codes = np.asarray(codes, dtype=np.uint8)
    scale = ue8m0_decode(scale_exp)
    N, K = codes.shape[-2], codes.shape[-1]
    rows = np.arange(N) // block
    cols = np.arange(K) // block
    per_elem = scale[..., rows[:, None], cols[None, :]]
    return fp8_e4m3_decode(codes) * per_elem


def moe_forward_fp8(x, Wr, bias, w13_q, w13_s, w2_q, w2_s, ws13_q, ws13_s, ws2_q, ws2_s,
                    cfg: MoeConfig, residual=None, ids=None, token_mask=None):
    """``moe_forward`` with FP8 expert weights: each weight matrix is the
    block dequantisation of its codes and scale exponents (``*_q`` uint8
    codes shaped like the bf16 weights, ``*_s`` uint8 scale exponents per
    128 x 128 block); everything else as ``moe_forward``."""
    deq = lambda q, sc: None if q is None else fp8_block_dequant(q, sc)
    return moe_forward(x, Wr, bias, deq(w13_q, w13_s), deq(w2_q, w2_s),
                       deq(ws13_q, ws13_s), deq(ws2_q, ws2_s), cfg,
                       residual=residual, ids=ids, token_mask=token_mask)


# ----------------------------------------------------------------------------
# RMSNorm for a residual stack of blocks ([S2]: RMSNorm accumulates in fp32)
# ----------------------------------------------------------------------------
def rmsnorm(x: np.ndarray, eps: float = 1e-6, gamma=None) -> np.ndarray:
    """x * rsqrt(mean(x^2) + eps) * gamma in float64 (gamma = 1 when None)."""
    xd = x.astype(np.float64)
    r = xd / np.sqrt(np.mean(xd * xd, axis=1, keepdims=True) + eps)
    if gamma is not None:
        r = r * gamma.astype(np.float64)[None, :]
    return r
