"""Algorithmic work of the scan and the update, and the B200 ceilings they meet.

Scan, per element (b, d, t):
  MUFU-class operations: 16 ex2 for Abar (one per state entry) + 2 for
  softplus (ex2 and a reciprocal, or ex2 and lg2 for bf16 inputs) + the silu
  gate (ex2 and a reciprocal, or one tanh for bf16 inputs) = 20 (fp32) or 19
  (bf16), plus one reciprocal of Delta with the zero-order hold.
  At 16 per clock per SM this is the binding pipe; the
  bytes (u, delta, z read, out written, plus each batch row's B and C shared
  by all channels) are about 8 per element in bf16, far below what HBM moves
  in the same time.
Update, per layer: the fp32 state is read and written once (2 x 64 bytes per
  chain at N = 16) next to a few bytes of token inputs, so HBM bandwidth
  bounds it.

The state-size arithmetic of "Mamba 与状态空间模型" (section 固定大小的状态) and
the KV-cache arithmetic of its section 越读越长的缓存 are reproduced by
``state_numbers`` and ``kv_cache_bytes_per_token`` (the tests pin both to the
page's printed figures).
"""
from __future__ import annotations

MUFU_PER_SM_PER_CLOCK = 16
EXP_PER_STATE = 1
SOFTPLUS_MUFU = 2
SILU_MUFU = 2
ZOH_MUFU = 1          # zero-order hold: 1 / Delta once per element


SILU_MUFU_BF16 = 1    # bf16 path: one tanh


def scan_mufu_per_element(dstate: int = 16, has_z: bool = True, softplus: bool = True,
                          zoh: bool = False, io_bytes: int = 4) -> int:
    """MUFU operations the scan kernel issues per element: one ex2 per state
    entry, softplus (ex2 + rcp for fp32 inputs, ex2 + lg2 for bf16), the gate
    (ex2 + rcp for fp32, one tanh for bf16) and 1/Delta with the zero-order hold."""
    silu = (SILU_MUFU_BF16 if io_bytes == 2 else SILU_MUFU) if has_z else 0
    return (dstate * EXP_PER_STATE + (SOFTPLUS_MUFU if softplus else 0) + silu
            + (ZOH_MUFU if zoh else 0))


def scan_mufu_method(dstate: int = 16, has_z: bool = True, softplus: bool = True,
                     zoh: bool = False) -> int:
    """MUFU operations per element that the method itself needs, independent
    of how a kernel evaluates them: one exponential per state entry for Abar,
    softplus as an exponential and a logarithm, the silu gate as an
    exponential and a reciprocal, and 1/Delta with the zero-order hold."""
    return (dstate * EXP_PER_STATE + (SOFTPLUS_MUFU if softplus else 0)
            + (SILU_MUFU if has_z else 0) + (ZOH_MUFU if zoh else 0))


def scan_bytes(batch: int, dim: int, dstate: int, seqlen: int, io_bytes: int = 2,
               bc_bytes: int = 2, has_z: bool = True, last_state: bool = False,
               start_state: bool = False) -> int:
    """HBM bytes one scan must move: u, delta, (z) read, out written, B and C
    read once per batch row, A/D/bias once, last_state written, the start
    state read."""
    elems = batch * dim * seqlen
    io = elems * io_bytes * (3 + (1 if has_z else 0))
    bc = 2 * batch * dstate * seqlen * bc_bytes
    params = dim * dstate * 4 + 2 * dim * 4
    tail = batch * dim * dstate * 4 if last_state else 0
    head = batch * dim * dstate * 4 if start_state else 0
    return io + bc + params + tail + head


def mufu_peak_elements_per_s(sm_count: int, sm_mhz: float, mufu_per_element: int) -> float:
    """Elements per second if every SM's MUFU pipe issued every clock."""
    return sm_count * MUFU_PER_SM_PER_CLOCK * sm_mhz * 1e6 / mufu_per_element


def update_bytes(batch: int, dim: int, dstate: int, io_bytes: int = 2, bc_bytes: int = 2,
                 has_z: bool = True) -> int:
    """HBM bytes of one state update: state read + written, x, dt, (z) read,
    out written, B and C, and the per-channel parameters."""
    chains = batch * dim
    state = 2 * chains * dstate * 4
    tok = chains * io_bytes * (3 + (1 if has_z else 0))
    bc = 2 * batch * dstate * bc_bytes
    params = dim * dstate * 4 + 2 * dim * 4
    return state + tok + bc + params


def state_numbers(layers: int, channels: int, dstate: int, conv_taps: int) -> int:
    """Numbers in a model's recurrent state: per layer and channel, dstate SSM
    entries plus the short convolution's last conv_taps inputs."""
    return layers * channels * (dstate + conv_taps)


def kv_cache_bytes_per_token(layers: int, width: int, bytes_per_number: int) -> int:
    """A Transformer's KV cache per token: a key and a value of `width`
    numbers in every layer."""
    return 2 * layers * width * bytes_per_number


def ssd_bytes(batch: int, seqlen: int, nheads: int, headdim: int = 64, ngroups: int = 1,
              dstate: int = 128, has_z: bool = True, initial_state: bool = False,
              final_state: bool = True) -> int:
    """HBM bytes of one Mamba-2 layer pass in bf16: x, (z), dt read and out
    written per (token, head); B and C once per (token, group); the fp32
    state read (start state) and written (final state) once per head."""
    tokens = batch * seqlen
    per_head = (2 + 2 + (2 if has_z else 0)) * headdim + 2
    state = batch * nheads * headdim * dstate * 4
    return (tokens * nheads * per_head + tokens * ngroups * dstate * 2 * 2 +
            state * (int(initial_state) + int(final_state)))


def ssd_chunk_flops(batch: int, seqlen: int, nheads: int, headdim: int = 64,
                    dstate: int = 128, chunk: int = 128) -> int:
    """Dense tensor-core FLOPs the chunked algorithm issues per pass: per chunk
    and head, C B^T (chunk x chunk x dstate), the masked matrix times x
    (chunk x chunk x headdim), the chunk's state B^T x (dstate x chunk x
    headdim) and the entering state's read-out C H^T (chunk x dstate x
    headdim), 2 FLOPs per multiply-add.  Chunks are counted whole (a ragged
    last chunk is padded)."""
    chunks = -(-seqlen // chunk)
    per = 2 * (chunk * chunk * dstate + chunk * chunk * headdim + 2 * dstate * chunk * headdim)
    return batch * nheads * chunks * per


def ssd_issued_flops(batch: int, seqlen: int, nheads: int, headdim: int = 64,
                     dstate: int = 128, chunk: int = 128) -> int:
    """Tensor-core FLOPs the Mamba-2 layer kernel issues per pass.  The three
    operands it computes (the masked matrix, the weighted input and the state
    copy) enter as bf16 hi/lo pairs, so the three products that take them are
    issued twice; C B^T, whose operands are inputs, once."""
    chunks = -(-seqlen // chunk)
    per = 2 * (chunk * chunk * dstate + 2 * (chunk * chunk * headdim + 2 * dstate * chunk * headdim))
    return batch * nheads * chunks * per
