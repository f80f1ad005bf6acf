"""The Swimba layer workloads this library is built and measured on.

Each workload fixes the layer's dimensions (notation of the Swimba paper,
"Swimba: Switch Mamba Model Scales State Space Models", arXiv 2603.06938,
Method section, key design 1): batch B, sequence length T, model width D,
H heads of head dimension P, SSM state dimension N, G groups for the B/C
streams, E experts of which k are active per token, and the SSD chunk length Q.

G = H throughout: the paper's notes give each expert its own B, C and x stream,
and "per head" is read as applying to all three, so every head carries its own
N-wide B and C.  The library also accepts any G dividing H.
"""
from dataclasses import dataclass, replace

F32 = "f32"
BF16 = "bf16"


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    d_model: int
    nheads: int
    headdim: int      # P
    dstate: int       # N
    n_experts: int    # E
    top_k: int        # k
    chunk: int        # Q
    dtype: str        # dtype of X, weights and y ("f32" or "bf16"); dt, pi and the state are fp32
    ngroups: int = 0  # G; 0 means G = H
    seed: int = 0
    prefill: int = 0  # decode workloads: prefill length that builds the cached state

    @property
    def G(self):
        return self.ngroups or self.nheads

    @property
    def M(self):
        return self.batch * self.seqlen

    @property
    def W_e(self):
        """Width of one expert's projection: x (H*P) + B (G*N) + C (G*N)."""
        return self.nheads * self.headdim + 2 * self.G * self.dstate

    def with_(self, **kw):
        return replace(self, **kw)


SEED0 = 0x5EED0000

TINY_F32 = Workload("tiny_f32", batch=1, seqlen=256, d_model=128, nheads=2, headdim=64, dstate=16,
                    n_experts=4, top_k=2, chunk=64, dtype=F32, seed=SEED0 + 0)
BASE = Workload("base_B4_T2048_D768_H24_E8_k2", batch=4, seqlen=2048, d_model=768, nheads=24, headdim=64,
                dstate=128, n_experts=8, top_k=2, chunk=256, dtype=BF16, seed=SEED0 + 1)


def esweep(E):
    """Expert-count sweep at fixed activity (k=2): the base layer with E experts."""
    return BASE.with_(name=f"esweep_E{E}", n_experts=E, seed=SEED0 + 2)


ESWEEP_E = (8, 16, 32, 64)
LONG = Workload("long_B1_T32768_D2048_H64_E16_k2", batch=1, seqlen=32768, d_model=2048, nheads=64, headdim=64,
                dstate=128, n_experts=16, top_k=2, chunk=256, dtype=BF16, seed=SEED0 + 3)
# Recurrent decode: 256 sequences, one new token each, cached fp32 state of H x N x P per sequence,
# the state built by a 512-token prefill.
DECODE = Workload("decode_B256_D2048_H64_E16_k2", batch=256, seqlen=1, d_model=2048, nheads=64, headdim=64,
                  dstate=128, n_experts=16, top_k=2, chunk=256, dtype=BF16, seed=SEED0 + 4, prefill=512)

# The base layer with B and C shared by groups of heads (G = H/4 and G = 1, Mamba-2 style groups).
BASE_G6 = BASE.with_(name="base_G6_B4_T2048_D768_H24_E8_k2", ngroups=6, seed=SEED0 + 5)
BASE_G1 = BASE.with_(name="base_G1_B4_T2048_D768_H24_E8_k2", ngroups=1, seed=SEED0 + 6)

ALL = {w.name: w for w in (TINY_F32, BASE, *(esweep(e) for e in ESWEEP_E), LONG, DECODE, BASE_G6, BASE_G1)}
