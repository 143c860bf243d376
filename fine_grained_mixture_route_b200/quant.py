"""FP8 (e4m3) weight format for the routed experts.

Each output channel (row of an nn.Linear weight [out, in]) gets one fp32 scale,
scale = max |w_row| / 448 (448 is the largest finite e4m3 value; an all-zero row gets scale 1),
and the codes are q = round-to-nearest-even_e4m3(w / scale).  The layer then computes with the
dequantized weights q * scale, which are exactly representable, so the fp64 oracle can run on
them directly.  Keeping the shared experts in bf16 follows the quantisation advice of the
DeepSeek-V2 explainer (eliteato.com/news/32734, §5.5): the always-on experts are the most
sensitive to quantisation error.

The conversion runs once, offline, in the library's per-row quantiser (moe_quantize_rows_e4m3,
the same kernel the FP8 layer uses for its activation rows): bf16 weights on the GPU in, codes
and scales out.  There is no other implementation of the format's arithmetic here.

The block-scaled variant (quantize_stack(..., fmt="mxfp8"), moe_quantize_weights_mx) keeps one
power-of-two scale per run of 32 inputs of each row instead of one per row: the per-group option
of the same §5.5 advice, in the form the sm_100a tensor cores apply inside the MMA.  The layer
then quantises the expert inputs and hidden rows in runs of 32 as well.
"""
from __future__ import annotations

from typing import Dict, Optional, Tuple

import torch

from fine_grained_mixture_route_b200 import moe

E4M3_MAX = 448.0


def quantize_rows(w: torch.Tensor, ws: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """w [..., out, in] bf16 on a CUDA device -> (codes [..., out, in] uint8, scales [..., out] fp32),
    by moe_quantize_rows_e4m3 (in must be a multiple of 8)."""
    if w.dtype != torch.bfloat16 or w.device.type != "cuda":
        raise ValueError("quantize_rows converts bf16 weights on a CUDA device (the library's e4m3 quantiser)")
    flat = w.reshape(-1, w.shape[-1]).contiguous()
    ws = torch.zeros(256, dtype=torch.uint8, device=w.device) if ws is None else ws
    codes, scales = moe.quantize_rows_e4m3(flat, ws)
    moe.check_device_error(ws)
    return codes.reshape(w.shape), scales.reshape(w.shape[:-1])


def dequantize_rows(q: torch.Tensor, scale: torch.Tensor) -> torch.Tensor:
    """codes uint8 + scales -> fp32 weights q * scale (for inspection; the layer never expands them)."""
    return q.view(torch.float8_e4m3fn).float() * scale.unsqueeze(-1)


def quantize_stack(stack: Dict[str, Optional[torch.Tensor]], fmt: str = "e4m3") -> Dict[str, Optional[torch.Tensor]]:
    """Routed expert stack (bf16 on the GPU: w1, w3 [E, I, d]; w2 [E, d, I]; biases unchanged) ->
    codes in w1/w3/w2 (uint8; w1 and w3 the two halves of one [2, E, I, d] buffer) and
    fmt "e4m3": per-row scales in s1, s3 [E, I] and s2 [E, d];
    fmt "mxfp8": block-scale bytes in sf13 (w1 and w3) and sf2 (w2), [E, bytes per expert] in the
    tiled order of include/moe.h."""
    if fmt == "mxfp8":
        return _quantize_stack_mx(stack)
    if fmt != "e4m3":
        raise ValueError('fmt must be "e4m3" or "mxfp8"')
    out = dict(stack)
    ws = torch.zeros(256, dtype=torch.uint8, device=stack["w1"].device)
    codes13 = None
    for w, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        q, sc = quantize_rows(stack[w], ws)
        if w in ("w1", "w3"):                 # W1 and W3 codes as the two halves of one buffer
            if codes13 is None:
                codes13 = torch.empty((2,) + tuple(q.shape), dtype=q.dtype, device=q.device)
            codes13[0 if w == "w1" else 1].copy_(q)
            out[w] = codes13[0 if w == "w1" else 1]
            del q
        else:
            out[w] = q
        out[sname] = sc
    return out


def _quantize_stack_mx(stack: Dict[str, Optional[torch.Tensor]]) -> Dict[str, Optional[torch.Tensor]]:
    w1, w3, w2 = stack["w1"], stack["w3"], stack["w2"]
    for w in (w1, w3, w2):
        if w.dtype != torch.bfloat16 or w.device.type != "cuda":
            raise ValueError("quantize_stack converts bf16 weights on a CUDA device")
    codes13 = torch.empty((2,) + tuple(w1.shape), dtype=torch.uint8, device=w1.device)
    _, _, sf13 = moe.quantize_weights_mx(moe.MX_UP, w1.contiguous(), w3.contiguous(), codes13[0], codes13[1])
    c2, _, sf2 = moe.quantize_weights_mx(moe.MX_DOWN, w2.contiguous())
    out = {k: v for k, v in stack.items() if k not in ("s1", "s3", "s2")}
    out.update(w1=codes13[0], w3=codes13[1], w2=c2, sf13=sf13, sf2=sf2)
    return out


def dequantize_stack(qstack: Dict[str, Optional[torch.Tensor]]) -> Dict[str, Optional[torch.Tensor]]:
    """The fp32 weights an FP8 stack stands for (biases unchanged)."""
    out = {k: v for k, v in qstack.items() if k not in ("s1", "s3", "s2")}
    for w, sname in (("w1", "s1"), ("w3", "s3"), ("w2", "s2")):
        out[w] = dequantize_rows(qstack[w], qstack[sname])
    return out
