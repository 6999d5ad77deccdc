"""State-dict export through one grouped launch of the export quantizer.

Host-side rules from "parameter-golf 16MB 极限压缩实战：11L MLP3x + Int6 QAT +
zstd-22 记录详解", section "后训练量化导出":
  - tensors that are not 2-D, or hold at most 65,536 elements
    (INT8_KEEP_FLOAT_MAX_NUMEL; "at most" is the reading taken), pass through
    as fp16;
  - the tied embedding passes through as fp16 (FP16_EMBED_EXPORT);
  - other 2-D tensors get per-row codes and fp16 scales: int6 when they
    belong to a block i with INT6_LAYER_START <= i <= INT6_LAYER_END (both
    inclusive, -1 = int6 off), else int8.
From "Depth Recurrence + Mixed-Precision Quant", reproduction commands
(MLP_INT5 / ATTN_INT5): with mlp_int5 every block MLP weight
("blocks.<i>.mlp."), with attn_int5 every block attention weight
("blocks.<i>.attn."), is exported on the int5 grid instead.
The per-row arithmetic all runs in the library's export kernel.
"""
import re

import torch

from . import qat

KEEP_FLOAT_MAX_NUMEL = 65536
_BLOCK = re.compile(r"^blocks\.(\d+)\.")


def export_mode(name, shape, numel, int6_range=(0, 10), embed_name="tok_emb.weight",
                mlp_int5=False, attn_int5=False):
    """Export mode of one tensor: 5, 6, 8 or qat.QAT_EXPORT_FP16."""
    if len(shape) != 2 or numel <= KEEP_FLOAT_MAX_NUMEL or name == embed_name:
        return qat.QAT_EXPORT_FP16
    m = _BLOCK.match(name)
    if m and ((mlp_int5 and ".mlp." in name) or (attn_int5 and ".attn." in name)):
        return 5
    start, end = int6_range
    if m and start >= 0 and end >= 0 and start <= int(m.group(1)) <= end:
        return 6
    return 8


def plan(state_dict, int6_range=(0, 10), embed_name="tok_emb.weight", mlp_int5=False,
         attn_int5=False):
    """(name, mode) for every tensor, in order."""
    return [(n, export_mode(n, tuple(t.shape), t.numel(), int6_range, embed_name, mlp_int5,
                            attn_int5))
            for n, t in state_dict.items()]


def export_state_dict(state_dict, int6_range=(0, 10), embed_name="tok_emb.weight", stream=None,
                      mlp_int5=False, attn_int5=False, pack6=False, clip_search=False):
    """Quantize a dict of fp32 CUDA tensors.  Returns name -> dict with
    kind 'int5'/'int6'/'int8' (codes int8 [rows,cols], scale16 fp16 [rows]) or
    kind 'fp16' (values fp16, original shape).  With pack6, int5 / int6 tensors
    hold 'packed' (uint8 [rows, cols*3/4], the 6-bit packed codes; see
    qat.unpack_codes6) in place of 'codes'.  clip_search: every quantized row
    keeps the clip quantile of least reconstruction error among the library's
    candidates (the leaderboard's "GPTQ-lite" clip search, read as a data-free
    per-row search).  Launches in chunks of at most
    QAT_EXPORT_MAX_DESCS descriptors (one launch for a state dict that fits)."""
    out = {}
    descs = []
    for name, mode in plan(state_dict, int6_range, embed_name, mlp_int5, attn_int5):
        t = state_dict[name]
        if t.dtype != torch.float32 or not t.is_contiguous():
            raise ValueError("%s: expected a contiguous fp32 tensor" % name)
        if mode == qat.QAT_EXPORT_FP16:
            v = torch.empty(t.shape, dtype=torch.float16, device=t.device)
            out[name] = {"kind": "fp16", "values": v}
            descs.append((t.reshape(-1), mode, v, None))
        else:
            rows, cols = t.shape
            s = torch.empty(rows, dtype=torch.float16, device=t.device)
            flags = qat.QAT_EXPORT_CLIP_SEARCH if clip_search else 0
            if pack6 and mode in (5, 6):
                p = torch.empty((rows, cols * 3 // 4), dtype=torch.uint8, device=t.device)
                out[name] = {"kind": "int%d" % mode, "packed": p, "scale16": s}
                descs.append((t, mode, p, s, flags | qat.QAT_EXPORT_PACK6))
            else:
                c = torch.empty((rows, cols), dtype=torch.int8, device=t.device)
                out[name] = {"kind": "int%d" % mode, "codes": c, "scale16": s}
                descs.append((t, mode, c, s, flags))
    for i in range(0, len(descs), qat.QAT_EXPORT_MAX_DESCS):
        qat.quantize_export_batch(descs[i:i + qat.QAT_EXPORT_MAX_DESCS], stream=stream)
    return out
