"""Expert parallelism over the ranks of one node ("MindIE-SD Fused MoE", execution flow:
dispatch, mlp, combine, and the dynamic dispatcher's all-to-all; "MATE Mega MoE", Typical Flow:
up to 8 intranode ranks).

Rank r of R owns experts r*E/R .. (r+1)*E/R - 1 and its own batch of tokens.  One step, on every
rank:

  1. route its tokens (``moe_route``);
  2. order its routed slots by destination rank and gather their token rows
     (``moe_ep_dispatch``);
  3. exchange the counts, then the rows and their local expert ids (all-to-all);
  4. run the rows it received through its experts, fp32 outputs in arrival order
     (``moe_forward_rows``);
  5. send the output rows back (the reverse all-to-all);
  6. combine them in slot order into bf16 (``moe_combine_rows``).

Every device step runs in the library's kernels; the exchange is ``torch.distributed``'s
all-to-all (NCCL over NVLink between GPUs, gloo in the CPU tests).  A row's expert output depends
only on its own row and its expert's weights, so each token's output is bit-identical to the
single-GPU ``forward``.

The device steps are taken from an ``ops`` object (``LibraryOps`` for the GPU library); the CPU
tests pass the oracle's versions of the same steps to check the exchange logic.
"""
from __future__ import annotations

from dataclasses import replace


class LibraryOps:
    """The device steps of an expert-parallel step, from libmoefp8.so."""

    rows_dtype = "float32"          # the expert side's output rows

    def __init__(self, moe_module=None):
        if moe_module is None:
            import mixture_experts_fp8_b200 as moe_module
        self.moe = moe_module
        self._rows_ws = {}          # device -> the expert side's workspace (grows, never shrinks)

    def rows_workspace(self, cfg_rows, device):
        """A workspace for the expert-side problem cfg_rows, kept from step to step: the row
        count varies per step, so the buffer grows to the largest problem seen and is reused (the
        steps run in stream order, so one buffer serves them all)."""
        need = self.moe.workspace_size(cfg_rows)
        ws = self._rows_ws.get(str(device))
        if ws is None or ws.numel() < need:
            ws = self.moe.new_workspace(cfg_rows, device)
            self._rows_ws[str(device)] = ws
        return ws

    def route(self, cfg, router_logits, per_expert_scale):
        return self.moe.route(cfg, router_logits, per_expert_scale=per_expert_scale)

    def dispatch(self, cfg, ranks, x, topk_idx, workspace):
        return self.moe.ep_dispatch(cfg, ranks, x, topk_idx, workspace)

    def rows(self, cfg_rows, rows, expert_of_row, weights_local, w13_bias, w2_bias):
        return self.moe.forward_rows(cfg_rows, rows, expert_of_row, weights_local, w13_bias=w13_bias,
                                     w2_bias=w2_bias, workspace=self.rows_workspace(cfg_rows, rows.device))

    def combine(self, cfg, o_rows, slot_pos, topk_weights, status=None):
        return self.moe.combine_rows(cfg, o_rows, slot_pos, topk_weights, status=status)

    def new_workspace(self, cfg, device):
        return self.moe.new_workspace(cfg, device)

    def status_word(self, workspace):
        """The dispatch's status word (device int32 [1]: the first word of the workspace)."""
        import torch
        return workspace[:4].view(torch.int32)


_LIBRARY_OPS = None


def _library_ops():
    """One LibraryOps per process, so that its expert-side workspace outlives a step."""
    global _LIBRARY_OPS
    if _LIBRARY_OPS is None:
        _LIBRARY_OPS = LibraryOps()
    return _LIBRARY_OPS


def rows_config(cfg, ranks: int, n_rows: int):
    """The expert side's problem: n_rows rows, one slot each, this rank's experts."""
    return replace(cfg, num_tokens=n_rows, top_k=1, num_experts=cfg.num_experts // ranks, routing=0,
                   renormalize=0, group_count=1, k_group=1, group_select_mode=0, routed_scaling_factor=1.0,
                   shared_experts=0)


def all_to_all_rows(dist, group, send, send_splits, recv_splits):
    """Rows of `send` (first dimension) to every rank by `send_splits`; returns the rows received,
    by rank, per `recv_splits`.  bf16 rows travel as int32 bit patterns (pairs of values), a type
    every backend moves."""
    import torch
    bf16 = send.dtype == torch.bfloat16
    flat = send.contiguous().view(torch.int32) if bf16 else send.contiguous()
    out = torch.empty((sum(recv_splits),) + tuple(flat.shape[1:]), dtype=flat.dtype, device=flat.device)
    dist.all_to_all_single(out, flat, recv_splits, send_splits, group=group)
    return out.view(torch.bfloat16) if bf16 else out


def ep_step(cfg, ranks: int, x, router_logits, weights_local, dist, group=None, ops=None, per_expert_scale=None,
            w13_bias_local=None, w2_bias_local=None, workspace=None):
    """One expert-parallel forward on this rank: its tokens x [T, H] (bf16) and router logits
    [T, E] in, y [T, H] (bf16) out.  cfg: this rank's tokens and the global expert count;
    weights_local: moe.transform_weights of this rank's E/R experts.  Returns (y, stats)."""
    import torch
    ops = ops or _library_ops()
    dev = x.device
    if workspace is None:
        workspace = ops.new_workspace(cfg, dev)
    idx, w = ops.route(cfg, router_logits, per_expert_scale)
    send_counts, send_x, send_expert, slot_pos = ops.dispatch(cfg, ranks, x, idx, workspace)

    # counts first (the splits of the row exchanges), then rows and ids, on the same device
    sc = send_counts.to(torch.int64)
    rc = torch.empty_like(sc)
    dist.all_to_all_single(rc, sc, group=group)
    status = ops.status_word(workspace) if hasattr(ops, "status_word") else None
    parts = [sc, rc] + ([status.to(torch.int64)] if status is not None else [])
    vals = [int(v) for v in torch.cat(parts).tolist()]   # one read-back: both split lists, the status
    send_splits, recv_splits = vals[:ranks], vals[ranks:2 * ranks]
    dispatch_status = vals[2 * ranks] if status is not None else 0
    recv_x = all_to_all_rows(dist, group, send_x[:sum(send_splits)], send_splits, recv_splits)
    recv_e = all_to_all_rows(dist, group, send_expert[:sum(send_splits)], send_splits, recv_splits)

    n = sum(recv_splits)
    if n > 0:
        o_recv = ops.rows(rows_config(cfg, ranks, n), recv_x, recv_e, weights_local, w13_bias_local,
                          w2_bias_local)
    else:                              # nothing routed to this rank's experts
        o_recv = torch.empty((0, cfg.hidden), dtype=getattr(torch, ops.rows_dtype), device=dev)
    o_home = all_to_all_rows(dist, group, o_recv, recv_splits, send_splits)
    y = ops.combine(cfg, o_home, slot_pos, w, status=status)
    if dispatch_status != 0:
        # every rank has taken the same collective steps; only now report the bad routing (a slot
        # whose expert id was out of range was not sent, and its token lacks that slot's term)
        from . import MoeError
        raise MoeError(dispatch_status, "moe_ep_dispatch: an expert id outside [0, num_experts) "
                                        "(status word MOE_ERR_BOUNDS); its slot was not sent")
    return y, {"sent": send_splits, "received": recv_splits}
