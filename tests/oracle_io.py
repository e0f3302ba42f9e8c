"""Turn generated decode inputs into the numpy arrays the oracle reads."""
import numpy as np
import torch

from oracle import mla_oracle as O


def to_numpy(inp):
    q = inp.q.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    blocks = inp.blocks.detach().cpu().numpy()
    scales = inp.scales.detach().cpu().numpy()
    L = (inp.cache_lengths.detach().cpu().to(torch.int64) & 0xFFFFFFFF).numpy()
    lut = (inp.lookup_table.detach().cpu().to(torch.int64) & 0xFFFFFFFF).numpy()
    slut = None
    if inp.scales_lookup_table is not None:
        slut = (inp.scales_lookup_table.detach().cpu().to(torch.int64) & 0xFFFFFFFF).numpy()
    return dict(q=q, blocks=blocks, scales=scales, cache_lengths=L, lookup_table=lut,
                scales_lookup_table=slut, max_prompt_length=inp.max_prompt_length,
                layer_idx=inp.layer_idx, softmax_scale=inp.softmax_scale)


def oracle_decode(inp, **kw):
    a = to_numpy(inp)
    return O.decode(a["q"], a["blocks"], a["scales"], a["cache_lengths"], a["lookup_table"],
                    a["scales_lookup_table"], a["max_prompt_length"], a["layer_idx"],
                    a["softmax_scale"], **kw)
