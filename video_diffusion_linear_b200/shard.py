"""Head sharding of the branch across ranks (one process per GPU).

Every step of the branch is per (batch, head): statistics, solve, both scans, gather and read-out
never mix heads.  A clip whose heads are split across ranks therefore needs no exchange inside the
branch: each rank runs vdn_branch_forward on its contiguous range of heads, with the per-head
parameters (text state, conv taps) of those heads and the shared ones (rms_w) whole.  Bringing a
sequence-sharded layout to a head-sharded one (the Ulysses all-to-all of q, k, v, gate and back)
belongs to the surrounding model, not to the branch.
"""
from __future__ import annotations


def head_range(H: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous, balanced range [h0, h1) of the H heads owned by `rank` of `world` (the first
    H % world ranks take one extra head; a rank may own none when world > H)."""
    if world < 1 or not 0 <= rank < world or H < 0:
        raise ValueError(f"bad shard: H={H} world={world} rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


PER_HEAD = {  # tensor -> axis of the head index
    "q": 2, "k": 2, "v": 2, "gate": 2, "beta": 2, "alpha": 2, "q_rope": 2, "k_rope": 2,
    "conv_k_w": 0, "conv_v_w": 0, "text_state": 0,
}


def shard_inputs(inputs: dict, world: int, rank: int) -> dict:
    """The rank's share of a synth-style input dict: per-head tensors restricted (and made
    contiguous, as the branch requires) to the rank's heads; shared tensors (rms_w) as they are."""
    H = inputs["q"].shape[2]
    h0, h1 = head_range(H, world, rank)
    out = {}
    for name, t in inputs.items():
        if t is None or name not in PER_HEAD:
            out[name] = t
            continue
        out[name] = t.narrow(PER_HEAD[name], h0, h1 - h0).contiguous()
    return out
