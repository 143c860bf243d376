"""FP8 (e4m3) weight format for the routed experts.

Each output channel (row of an nn.Linear weight [out, in]) gets one fp32 scale,
scale = max |w_row| / 448 (448 is the largest finite e4m3 value; an all-zero row gets scale 1),
and the codes are q = round-to-nearest-even_e4m3(w / scale).  The layer then computes with the
dequantized weights q * scale, which are exactly representable, so the fp64 oracle can run on
them directly.  Keeping the shared experts in bf16 follows the quantisation advice of the
DeepSeek-V2 explainer (eliteato.com/news/32734, §5.5): the always-on experts are the most
sensitive to quantisation error.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

E4M3_MAX = 448.0


def quantize_rows(w: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """w [..., out, in] (any float dtype) -> (codes [..., out, in] uint8, scales [..., out] fp32)."""
    wf = w.float()
    amax = wf.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    q = (wf / scale.unsqueeze(-1)).to(torch.float8_e4m3fn)
    return q.view(torch.uint8), scale.contiguous()


def dequantize_rows(q: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """codes uint8 + scales -> fp32 weights q * scale."""
    return q.view(torch.float8_e4m3fn).float() * scale.unsqueeze(-1)


def quantize_stack(stack: Dict[str, Optional[torch.Tensor]]) -> Dict[str, Optional[torch.Tensor]]:
    """Routed expert stack (w1, w3 [E, I, d]; w2 [E, d, I]; biases unchanged) -> codes in
    w1/w3/w2 (uint8; w1 and w3 the two halves of one [2, E, I, d] buffer) and per-row scales in
    s1, s3 [E, I] and s2 [E, d]."""
    out = dict(stack)
    codes13 = None
    for w, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = quantize_rows(stack[w])
        if w in ("w1", "w3"):                 # W1 and W3 codes as the two halves of one buffer
            if codes13 is None:
                codes13 = torch.empty((2,) + tuple(q.shape), dtype=q.dtype, device=q.device)
            codes13[0 if w == "w1" else 1].copy_(q)
            out[w] = codes13[0 if w == "w1" else 1]
        else:
            out[w] = q.contiguous()
        out[sname] = sc
    return out


def dequantize_stack(qstack: Dict[str, Optional[torch.Tensor]]) -> Dict[str, Optional[torch.Tensor]]:
    """The fp32 weights an FP8 stack stands for (biases unchanged)."""
    out = {k: v for k, v in qstack.items() if k not in ("s1", "s3", "s2")}
    for w, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        out[w] = dequantize_rows(qstack[w], qstack[sname])
    return out
