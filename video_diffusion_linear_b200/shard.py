"""Sharding of the branch across ranks (one process per GPU): by heads, and by frames (below).

Every step of the branch is per (batch, head): statistics, solve, both scans, gather and read-out
never mix heads, and neither does the windowed softmax branch.  A clip whose heads are split across
ranks therefore needs no exchange in the forward: each rank runs the unchanged entry points on its
contiguous range of heads, with the per-head parameters (text state, conv taps) of those heads and
the shared ones (rms_w) whole.  The backward's one exchange is the gradient of rms_w, which every
head shares: each rank's call sums it over its own heads, and reduce_shared_grads sums those
partials across the ranks.  Bringing a sequence-sharded layout to a head-sharded one (the Ulysses
all-to-all of q, k, v, gate and back) belongs to the surrounding model, not to the branch.
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


PER_HEAD = {  # tensor -> axis of the head index (inputs, the upstream gradient and the gradients)
    "q": 2, "k": 2, "v": 2, "gate": 2, "beta": 2, "alpha": 2, "q_rope": 2, "k_rope": 2, "dout": 2,
    "conv_k_w": 0, "conv_v_w": 0, "text_state": 0,
    "dq": 2, "dk": 2, "dv": 2, "dgate": 2, "dbeta": 2, "dalpha": 2,
    "dconv_k_w": 0, "dconv_v_w": 0, "dtext_state": 0,
}

SHARED_GRADS = ("drms_w",)  # gradients of parameters every head shares: summed across the ranks


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


def reduce_shared_grads(grads: dict, group=None) -> dict:
    """Sum the gradients of the shared parameters (rms_w) over the ranks of `group`, in place, with
    one all-reduce each (NCCL for CUDA tensors).  Per-head gradients stay on their rank.  A no-op
    without an initialised process group of more than one rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return grads
    for name in SHARED_GRADS:
        if grads.get(name) is not None:
            dist.all_reduce(grads[name], op=dist.ReduceOp.SUM, group=group)
    return grads


# ----------------------------------------------------------------------------- frame sharding
# For clips too long for one GPU the frames split instead.  Every frame's statistics, solve and
# read-out are local; the only coupling is the pair of scans.  Each rule's step is affine in the
# state, S_out = S_in G_f + B'_f, so a rank's run of frames composes into one map per direction,
# and the ranks before it (after it, for the suffix scan) fold into the seed it starts from.  A
# window then reads the prefix state just before it and the suffix state just after it, which can
# lie on another rank: those boundary states make the second, equally small exchange.  The
# functions below fix who owns which frames and which states cross; the arithmetic runs on the
# device.
#
# The device path (vdn_frames_maps / vdn_frames_finish) takes the exchange one step further: each
# rank publishes the affine map of every one of its chunks (not one per rank), so after a single
# all-gather every rank folds the maps into every chunk-edge state itself, and no state needs a
# second exchange.  frame_sharded_forward runs that sequence.

def _window(t: int, F: int, chunk: int, radius: int) -> tuple[int, int]:
    # chunk-aligned window of query frame t: its chunk widened by `radius` chunks each side
    c = t // chunk
    return max(0, chunk * (c - radius)), min(F - 1, chunk * (c + radius + 1) - 1)


def frame_range(F: int, world: int, rank: int, chunk: int) -> tuple[int, int]:
    """Frames [f0, f1) of `rank` under frame sharding: a contiguous run of whole chunks of `chunk`
    frames (the clip's last chunk may be short), the chunks split as head_range splits heads."""
    if chunk < 1 or F < 0:
        raise ValueError(f"bad frame shard: F={F} chunk={chunk}")
    c0, c1 = head_range(-(-F // chunk), world, rank)
    return min(F, c0 * chunk), min(F, c1 * chunk)


def remote_states(F: int, chunk: int, radius: int, f0: int, f1: int) -> tuple[list[int], list[int]]:
    """(pre, suf): the frames f whose prefix state P_f (read at lo - 1) and suffix state Q_f (read at
    hi + 1) the windows of query frames [f0, f1) need and another rank computes.  A window at a
    clip edge reads the seed and needs nothing."""
    pre, suf = set(), set()
    for t in range(f0, f1):
        lo, hi = _window(t, F, chunk, radius)
        if lo > 0 and not f0 <= lo - 1 < f1:
            pre.add(lo - 1)
        if hi < F - 1 and not f0 <= hi + 1 < f1:
            suf.add(hi + 1)
    return sorted(pre), sorted(suf)


def published_states(F: int, world: int, rank: int, chunk: int, radius: int) -> tuple[list[int], list[int]]:
    """(pre, suf): the frames of `rank` whose prefix / suffix states some other rank's windows read,
    i.e. what `rank` contributes to the boundary exchange."""
    f0, f1 = frame_range(F, world, rank, chunk)
    pre, suf = set(), set()
    for r in range(world):
        if r != rank:
            p, s = remote_states(F, chunk, radius, *frame_range(F, world, r, chunk))
            pre.update(f for f in p if f0 <= f < f1)
            suf.update(f for f in s if f0 <= f < f1)
    return sorted(pre), sorted(suf)


TOKEN_AXIS = {"q": 1, "k": 1, "v": 1, "gate": 1, "beta": 1, "q_rope": 1, "k_rope": 1, "dout": 1}


def frame_inputs(inputs: dict, F: int, world: int, rank: int, chunk: int) -> dict:
    """The rank's share of a synth-style input dict under frame sharding: the tokens of its frames
    (q, k, v, gate, beta, ...), alpha of its frames, and alpha of the whole clip as "alpha_all";
    per-head and shared parameters as they are."""
    f0, f1 = frame_range(F, world, rank, chunk)
    S = inputs["q"].shape[1] // F
    out = {}
    for name, t in inputs.items():
        if t is not None and name in TOKEN_AXIS:
            out[name] = t.narrow(TOKEN_AXIS[name], f0 * S, (f1 - f0) * S).contiguous()
        elif name == "alpha":
            out[name] = t.narrow(1, f0, f1 - f0).contiguous()
            out["alpha_all"] = t
        else:
            out[name] = t
    return out


def frame_sharded_forward(local: dict, F: int, world: int, rank: int, *, rule="vdn_solve", c=1.0, chunk=5,
                          radius=1, group=None, stream=None, check_status=True):
    """The branch output of this rank's frames (device tensors from frame_inputs): its chunk maps,
    one all-gather of every rank's maps (NCCL for CUDA tensors; none with one rank), then the fold,
    gather and read-out of its frames.  Both phases share one workspace, so its device status word
    reports an expired bounded wait of either phase; with check_status (CUDA tensors only) it is
    read after phase 2 (a synchronisation) and a timeout raises."""
    from . import api
    ws = None
    if local["k"].is_cuda:
        import torch
        f0, f1 = frame_range(F, world, rank, chunk)
        shape = api.shape_from(local["k"], f1 - f0, local.get("conv_k_w"))
        ws = torch.empty(api.frames_workspace_size(shape, F, world, rank, rule, chunk), dtype=torch.uint8,
                         device=local["k"].device)
    maps = api.frames_maps(local["k"], local["v"], local["beta"], local["alpha"], local.get("conv_k_w"),
                           local.get("conv_v_w"), F_total=F, world=world, rank=rank, rule=rule, c=c, chunk=chunk,
                           workspace=ws, stream=stream)
    if world > 1:
        import torch
        import torch.distributed as dist
        maps_all = torch.empty(world * maps.numel(), dtype=maps.dtype, device=maps.device)
        dist.all_gather_into_tensor(maps_all, maps, group=group)
    else:
        maps_all = maps
    out = api.frames_finish(local["q"], local["alpha_all"], local["gate"], local["rms_w"], local.get("text_state"),
                            maps_all, F_total=F, world=world, rank=rank, rule=rule, c=c, chunk=chunk, radius=radius,
                            workspace=ws, stream=stream)
    if ws is not None and check_status:
        api.check(api.workspace_status(ws, stream), "device status word after the frame-sharded branch")
    return out
