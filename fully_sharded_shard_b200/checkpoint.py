"""Save and restore one parameter group's sharded training state.

The state of a group is its fp32 master, m and v shards ([N][S] each, rank
major) and the AdamW step count.  They are written as one raw little-endian
fp32 file per buffer plus a small JSON header (shapes, N, S, step), so a
multi-step run can stop after any step and resume with the same bits.  The
layout is the library's: rank r's shard of parameter i at r*S + off_i.
"""
from __future__ import annotations

import json
import os
from typing import Sequence

import numpy as np
import torch

FORMAT = "fsdpk-group-state-v1"


def save_group_state(path: str, shapes: Sequence[Sequence[int]], world_size: int, S: int,
                     step: int, master: torch.Tensor, m: torch.Tensor, v: torch.Tensor) -> None:
    os.makedirs(path, exist_ok=True)
    n = world_size * S
    for name, t in (("master", master), ("m", m), ("v", v)):
        assert t.dtype == torch.float32 and t.numel() >= n, name
        t[:n].detach().cpu().numpy().astype("<f4").tofile(os.path.join(path, name + ".f32"))
    header = {"format": FORMAT, "shapes": [list(s) for s in shapes], "world_size": world_size,
              "S": S, "step": int(step)}
    with open(os.path.join(path, "header.json"), "w") as f:
        json.dump(header, f)


def load_group_state(path: str, shapes: Sequence[Sequence[int]], world_size: int, S: int,
                     master: torch.Tensor, m: torch.Tensor, v: torch.Tensor) -> int:
    """Fill master/m/v from `path`; return the step count.  The saved group must
    have the same shapes, world size and S."""
    with open(os.path.join(path, "header.json")) as f:
        header = json.load(f)
    if header.get("format") != FORMAT:
        raise ValueError(f"{path}: not a {FORMAT} checkpoint")
    if ([list(s) for s in shapes] != header["shapes"] or header["world_size"] != world_size
            or header["S"] != S):
        raise ValueError(f"{path}: saved for a different group layout")
    n = world_size * S
    for name, t in (("master", master), ("m", m), ("v", v)):
        data = np.fromfile(os.path.join(path, name + ".f32"), dtype="<f4")
        if data.size != n:
            raise ValueError(f"{path}/{name}.f32: {data.size} values, expected {n}")
        t[:n].copy_(torch.from_numpy(data.astype(np.float32)))
    return int(header["step"])
