"""Tensor-parallel use of the NVFP4 path over torch.distributed.

Every NVFP4 tensor carries one FP32 tensor scale over all of its elements
(NVFP4 wiki page, section "技術原理": the second, per-tensor level of the
two-level scaling).  Sharding the path over G ranks therefore needs exactly
one exchange where a quantized tensor is split: the ranks agree on its amax
(an all-reduce MAX of one float) before any block is encoded.

- Column-parallel GEMM (each rank holds N/G rows of W, x replicated): the
  ranks' outputs are the column blocks of y; no exchange.
- A tensor split by rows: ``quantize_row_sharded`` -- first pass on each
  rank (``nvfp4_amax``), all-reduce MAX of the amax, second pass with the
  shared amax (``nvfp4_quantize_with_amax``).  Each rank's codes and scales
  equal those rows of the whole tensor quantized at once.
- The MLP (``mlp_tensor_parallel``): gate and up column-parallel, so each
  rank holds a column block of h = SiLU(gate)*up; h's amax is all-reduced
  (MAX) before h is quantized, which keeps every 16-value block whole when the
  block width is a multiple of 16; the down projection is row-parallel on its
  K (each rank holds the matching column block of W_down), and the partial
  outputs are all-reduced (SUM).

The collectives run on whatever backend the process group has (NCCL on
GPUs; gloo goes through a host copy).  Every rank makes the same collective
calls in the same order.  All arithmetic stays in the library's kernels; this
module only sequences the calls.
"""
from __future__ import annotations


def _nv():
    import nvfp4_block_scaled_21_b200 as nv
    return nv


def _collective(t, op, group):
    """All-reduce t in place with op; through a host copy when the backend
    cannot take device tensors (gloo)."""
    import torch.distributed as dist
    if not t.is_cuda or dist.get_backend(group) == "nccl":
        dist.all_reduce(t, op=op, group=group)
        return t
    host = t.cpu()
    dist.all_reduce(host, op=op, group=group)
    t.copy_(host)
    return t


def allreduce_amax_(amax, group=None):
    """The one exchange of a sharded quantization: amax (one fp32) <- the
    largest over the ranks, in place."""
    import torch.distributed as dist
    return _collective(amax, dist.ReduceOp.MAX, group)


def quantize_row_sharded(x_shard, out, ws, group=None, lib=None, stream=None):
    """Quantize this rank's rows of a tensor split across the group by rows.

    x_shard: this rank's [rows_r][cols] bf16/fp32 CUDA tensor; out: an
    NVFP4Tensor of the same shape; ws: a workspace for NVFP4_OP_QUANTIZE.
    After the call every rank's out.tensor_scale is the whole tensor's and
    its codes and scales are those of its rows of the whole tensor."""
    import torch
    nv = lib or _nv()
    amax = torch.empty(1, dtype=torch.float32, device=x_shard.device)
    nv.nvfp4_amax(x_shard, amax, ws, stream)
    allreduce_amax_(amax, group)
    nv.nvfp4_quantize_with_amax(x_shard, amax, out, ws, stream)
    return out


def linear_column_parallel(x, w_shard, ws, y=None, lib=None):
    """y_r = x . W_r^T (bf16) for this rank's rows W_r of W: the column block
    r of the full y.  No exchange (gather the blocks only if the consumer
    needs all of y)."""
    import torch
    nv = lib or _nv()
    if y is None:
        y = torch.empty((x.shape[0], w_shard.rows), dtype=torch.bfloat16, device=x.device)
    nv.nvfp4_linear_fused(x, w_shard, ws, nv.EPI_STORE, y=y)
    return y


def mlp_tensor_parallel(x, wg_shard, wu_shard, wd_shard, group=None, lib=None):
    """y = down(quantize(SiLU(x Wg^T) * (x Wu^T))) with gate/up split by
    output rows (this rank: wg_shard, wu_shard, [N/G][K]) and down split by
    its reduction columns to match (this rank: wd_shard, [K_out][N/G]).

    Steps on each rank: the fused gate/up call writes h_r (fp32, this rank's
    column block of h); nvfp4_amax(h_r); all-reduce MAX; h_r quantized with
    the shared amax; y_r = h_q_r . Wd_r^T in fp32; all-reduce SUM of y_r.
    N/G must be a multiple of 16 so that no block of h straddles two ranks.
    Returns y (fp32, [M][K_out])."""
    import torch
    import torch.distributed as dist
    nv = lib or _nv()
    M, K = x.shape
    n_r = wg_shard.rows
    if n_r % 16:
        raise ValueError("mlp_tensor_parallel: each rank's share of the hidden size must be a multiple of 16")
    dev = x.device
    h = torch.empty((M, n_r), dtype=torch.float32, device=dev)
    h_q_local = nv.NVFP4Tensor.empty(M, n_r)       # the fused call's own (per-rank) quantization, not used
    ws_gu = nv.workspace(nv.OP_LINEAR_FUSED_SILU, M, n_r, K)
    nv.nvfp4_linear_fused(x, wg_shard, ws_gu, nv.EPI_SILU_MUL_REQUANT, y=h, w_up=wu_shard, y_q=h_q_local)
    h_q = nv.NVFP4Tensor.empty(M, n_r)
    quantize_row_sharded(h, h_q, nv.workspace(nv.OP_QUANTIZE, M, 0, n_r), group=group, lib=nv)
    y = torch.empty((M, wd_shard.rows), dtype=torch.float32, device=dev)
    nv.nvfp4_gemm(h_q, wd_shard, y, nv.workspace(nv.OP_GEMM, M, wd_shard.rows, n_r))
    _collective(y, dist.ReduceOp.SUM, group)
    return y
