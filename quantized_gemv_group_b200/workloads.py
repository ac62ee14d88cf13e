"""Shapes, bit schedules and byte counts of the decode workloads.

Host-side tables only; no kernel arithmetic.

* Llama-2-70B decoder block (grouped-query attention, 8 KV heads x 128):
  q/o 8192->8192, k/v 8192->1024, gate/up 8192->28672, down 28672->8192.
  Eighty such blocks plus two 32000 x 8192 embeddings and the RMSNorm
  vectors make 68,976,648,192 parameters, i.e. 137.95 GB in fp16, the
  figure "70B en 4GB de VRAM: la compresión neural de 2026, ¿es real?"
  (section "1. NanoQuant — sub-1-bit PTQ", bullet "Versión v3") quotes for
  Llama2-70B.
* Per-layer bit allocation: "TurboQuant: cuantizar modelos grandes para que
  quepan en local", section "Asignación de bits por capa" gives 5-6 bits to
  attention and 2 bits to MLP, averaging 2.7-3.2 bits per weight.  The fixed
  schedule below keeps attention at 6 bits in the first and last eight layers
  and 5 elsewhere, and MLP at 3 bits on even and 2 on odd layers (2.976
  code bits per weight).
* Binary low-rank rank: r = 32 * round(bpw * d_out * d_in / (32 (d_out + d_in))),
  so that r (d_out + d_in) / (d_out d_in) is the target bits per weight.
"""
from dataclasses import dataclass

HIDDEN = 8192
INTERMEDIATE = 28672
KV_DIM = 1024
N_LAYERS = 80
VOCAB = 32000

PROJS = ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj")
ATTN = ("q_proj", "k_proj", "v_proj", "o_proj")


@dataclass(frozen=True)
class Linear:
    name: str
    d_in: int   # k
    d_out: int  # n


def block_linears():
    return [
        Linear("q_proj", HIDDEN, HIDDEN),
        Linear("k_proj", HIDDEN, KV_DIM),
        Linear("v_proj", HIDDEN, KV_DIM),
        Linear("o_proj", HIDDEN, HIDDEN),
        Linear("gate_proj", HIDDEN, INTERMEDIATE),
        Linear("up_proj", HIDDEN, INTERMEDIATE),
        Linear("down_proj", INTERMEDIATE, HIDDEN),
    ]


def llama2_70b_params() -> int:
    per_layer = sum(l.d_in * l.d_out for l in block_linears()) + 2 * HIDDEN
    return N_LAYERS * per_layer + 2 * VOCAB * HIDDEN + HIDDEN


def schedule_bits(layer: int, proj: str, n_layers: int = N_LAYERS) -> int:
    """Fixed per-layer bit allocation (attention 5-6 bits, MLP 2-3 bits)."""
    if proj in ATTN:
        return 6 if (layer < 8 or layer >= n_layers - 8) else 5
    return 3 if layer % 2 == 0 else 2


def schedule_code_bits_per_weight(n_layers: int = N_LAYERS) -> float:
    tot_w = 0
    tot_b = 0
    for layer in range(n_layers):
        for l in block_linears():
            w = l.d_in * l.d_out
            tot_w += w
            tot_b += w * schedule_bits(layer, l.name, n_layers)
    return tot_b / tot_w


def group_packed_bytes(n: int, k: int, bits: int, group: int) -> int:
    """Codes plus one fp16 scale and one fp16 zero per group."""
    return n * k * bits // 8 + 4 * n * (k // group)


def group_bpw(bits: int, group: int) -> float:
    return bits + 32.0 / group


def binlr_rank(d_out: int, d_in: int, bpw: float) -> int:
    return 32 * int(round(bpw * d_out * d_in / (32.0 * (d_out + d_in))))


def binlr_bpw(d_out: int, d_in: int, r: int, with_scales: bool = False) -> float:
    b = r * (d_out + d_in) / (d_out * d_in)
    if with_scales:
        b += 16.0 * (d_out + d_in) / (d_out * d_in)
    return b


def binlr_bytes(d_out: int, d_in: int, r: int) -> int:
    """Sign bits of U and V plus fp16 s1, s2."""
    return r * (d_out + d_in) // 8 + 2 * (d_out + d_in)


def gemv_algorithmic_bytes(n: int, k: int, bits: int, group: int, M: int, x_bytes: int = 2) -> int:
    """Packed weights + scales/zeros + activations in + outputs out."""
    return group_packed_bytes(n, k, bits, group) + x_bytes * M * k + 2 * M * n


def binlr_algorithmic_bytes(d_out: int, d_in: int, r: int, M: int) -> int:
    return binlr_bytes(d_out, d_in, r) + 2 * M * (d_in + d_out)


BINLR_SHAPES = [(8192, 8192), (1024, 8192), (28672, 8192), (8192, 28672)]  # (d_out, d_in)
BINLR_BPW = (0.55, 0.8, 1.0)
