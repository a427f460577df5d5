"""Memory and communication accounting of data-parallel training -- TEST
INFRASTRUCTURE ONLY (part of the oracle).

Restated from the pages:
  * "CS336 lecture 8, parallelism basics", core concepts: mixed-precision
    Adam costs 2 (bf16 param) + 2 (bf16 grad) + 4 (fp32 master) + 4 + 4
    (Adam moments) = 16 bytes per parameter; ZeRO stage 1 needs
    (4 + K / N_gpu) bytes per parameter (K = optimizer-state bytes); its
    communication is 2 x #params, like DDP's all-reduce; stage 3 moves
    3 x #params.  FSDP section: the "does it fit" table at 12 bytes per
    parameter (K = 8) on 8 x A100-80G.
  * "DDP -> ZeRO -> TP/PP/CP" blog, section 1.1 and 3.1: 7B model, 14 + 14 + 84
    = 112 GB; per card at 64 cards ZeRO-1 ~29.3 GB, ZeRO-2 ~15.5 GB, ZeRO-3
    ~1.7 GB; section 2.2: ring all-reduce moves 2(N-1)/N of the gradient per
    card, ~28 GB per step for a 14 GB bf16 gradient.
Units: bytes and parameter counts are plain numbers; "GB" here is 1e9 bytes,
as the pages use it.
"""

PARAM_BYTES = 2        # bf16 parameter
GRAD_BYTES = 2         # bf16 gradient
MASTER_BYTES = 4       # fp32 master weight
MOMENT_BYTES = 4       # each of Adam's m and v, fp32


def bytes_per_param_mixed_adamw() -> int:
    return PARAM_BYTES + GRAD_BYTES + MASTER_BYTES + 2 * MOMENT_BYTES


def optimizer_state_bytes_per_param() -> int:
    """K: fp32 master + m + v."""
    return MASTER_BYTES + 2 * MOMENT_BYTES


def ddp_bytes_per_card(params, k=None):
    k = optimizer_state_bytes_per_param() if k is None else k
    return (PARAM_BYTES + GRAD_BYTES + k) * params


def zero1_bytes_per_card(params, n_gpu, k=None):
    """Optimizer state sharded: 2 + 2 + K / N bytes per parameter."""
    k = optimizer_state_bytes_per_param() if k is None else k
    return (PARAM_BYTES + GRAD_BYTES) * params + k * params / n_gpu


def zero2_bytes_per_card(params, n_gpu, k=None):
    """Optimizer state and gradients sharded: 2 + (2 + K) / N."""
    k = optimizer_state_bytes_per_param() if k is None else k
    return PARAM_BYTES * params + (GRAD_BYTES + k) * params / n_gpu


def zero3_bytes_per_card(params, n_gpu, k=None):
    """Everything sharded: (2 + 2 + K) / N."""
    k = optimizer_state_bytes_per_param() if k is None else k
    return (PARAM_BYTES + GRAD_BYTES + k) * params / n_gpu


def largest_model_that_fits(mem_bytes, n_gpu, stage, k):
    """Parameter count whose per-card state fills ``mem_bytes`` (activations
    ignored), for stage 0 (plain DDP) to 3."""
    per_param = {
        0: ddp_bytes_per_card(1, k),
        1: zero1_bytes_per_card(1, n_gpu, k),
        2: zero2_bytes_per_card(1, n_gpu, k),
        3: zero3_bytes_per_card(1, n_gpu, k),
    }[stage]
    return mem_bytes / per_param


def ring_allreduce_bytes_per_rank(n_elems, world_size, elem_bytes):
    """Reduce-scatter then all-gather around a ring: 2 (W-1) steps of 1/W."""
    return 2 * (world_size - 1) * (n_elems * elem_bytes) / world_size


def reduce_scatter_bytes_per_rank(n_elems, world_size, elem_bytes):
    return (world_size - 1) * (n_elems * elem_bytes) / world_size


def all_gather_bytes_per_rank(n_elems, world_size, elem_bytes):
    return (world_size - 1) * (n_elems * elem_bytes) / world_size


def zero1_comm_elems(params):
    """Reduce-scatter (#params) + all-gather (#params), the large-W limit."""
    return 2 * params


def zero3_comm_elems(params):
    """Two parameter all-gathers (forward, backward) + one gradient reduce-scatter."""
    return 3 * params
