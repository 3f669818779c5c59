"""Seeded synthetic inputs for the product-key memory lookup.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic.  Both the CUDA path and the CPU oracle consume the
same tensors made here.

Workloads (shapes and distributions follow the configurations the lookup is
measured on; all data is synthetic, no dataset is involved):

* ``tiny``     fp32, T=512, H=1, d_half=128, n_sub=32 (N=1024), k=8, d_v=256,
               seed 0.
* ``pkm``      bf16, T=8192 (4 x 2048), H=4, d_half=512, n_sub=1024
               (N=1,048,576), k=32, d_v=2048 (4 GiB value table).
* ``memplus``  bf16, T=16384, H=4, d_half=512, n_sub=4096 (N=16,777,216),
               k=32, d_v=d_model=1024 (32 GiB table), gate x W1, W2.
* ``train``    the ``pkm`` shapes plus an upstream gradient, with sub-keys
               biased towards a shared direction so that selected rows follow
               a Zipf popularity: (alpha, beta, gamma) = (0.5, 4.0, 4.9) were
               calibrated so that a least-squares fit of log(count) against
               log(rank) over ranks 1..10^4 of the selected rows gives an
               exponent of 1.10 (about 1.3e5 distinct rows of 2^20 slots).
* ``memplus_train``  the ``memplus`` shapes and tables plus an upstream
               gradient of the layer output (the Memory+ training step).
* ``decode``   8 tokens per step x 256 steps against the ``memplus`` tables.
* ``engram``   (``EngramWorkload``) the hashed n-gram lookup: 8 sequences x
               2048 tokens, 2- and 3-grams with 4 hash heads each, one table
               per head of 1,048,573 .. 1,048,433 rows (the eight largest
               primes below 2^20; 8.4 M rows x 1024 bf16 = 17 GB stacked),
               token ids uniform over 2^17 (so rows are spread over the
               tables; text would repeat n-grams), hidden state N(0,1).

Distributions: queries N(0,1); sub-keys N(0, std 1/sqrt(d_half)); values
N(0, std 0.02); x N(0,1); W1, W2 N(0, std 1/sqrt(1024)); upstream gradient
N(0,1).  The second parameter of N(.,.) is read as a standard deviation.
Small tensors are drawn on the CPU generator in fp32 and rounded to the
storage dtype (round to nearest even); value tables larger than 64 MiB are
drawn on the device generator in row chunks.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    d_half: int
    n_sub: int
    k: int
    d_v: int
    dtype: str  # "f32" or "bf16"
    seed: int
    memplus: bool = False
    d_model: int = 0
    train: bool = False
    decode_steps: int = 0
    # Zipf bias of the sub-keys (train workload): K[h,c,a] += beta*(rank+1)^-alpha * e,
    # queries += gamma * e, with e a fixed random unit vector per (h, c).
    zipf_alpha: float = 0.0
    zipf_beta: float = 0.0
    zipf_gamma: float = 0.0
    # seed of the parameter tables (sub-keys, values, W1, W2); defaults to seed
    table_seed_: int = -1

    @property
    def table_seed(self) -> int:
        return self.seed if self.table_seed_ < 0 else self.table_seed_

    @property
    def N(self) -> int:
        return self.n_sub * self.n_sub

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def d_out(self) -> int:
        return self.d_model if self.memplus else self.d_v

    def scaled(self, **kw) -> "Workload":
        """Same distributions at other sizes (for tests)."""
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        d = dict(workload=self.name, tokens=self.T, heads=self.H, d_half=self.d_half,
                 n_sub=self.n_sub, N=self.N, k=self.k, d_v=self.d_v, dtype=self.dtype)
        if self.memplus:
            d["d_model"] = self.d_model
        if self.decode_steps:
            d["decode_steps"] = self.decode_steps
        return d


WORKLOADS = {
    "tiny": Workload("tiny", T=512, H=1, d_half=128, n_sub=32, k=8, d_v=256,
                     dtype="f32", seed=0),
    "pkm": Workload("pkm", T=8192, H=4, d_half=512, n_sub=1024, k=32, d_v=2048,
                    dtype="bf16", seed=1002),
    "memplus": Workload("memplus", T=16384, H=4, d_half=512, n_sub=4096, k=32,
                        d_v=1024, dtype="bf16", seed=1003, memplus=True, d_model=1024),
    "train": Workload("train", T=8192, H=4, d_half=512, n_sub=1024, k=32, d_v=2048,
                      dtype="bf16", seed=1004, train=True,
                      zipf_alpha=0.5, zipf_beta=4.0, zipf_gamma=4.9),
    "memplus_train": Workload("memplus_train", T=16384, H=4, d_half=512, n_sub=4096, k=32,
                              d_v=1024, dtype="bf16", seed=1006, memplus=True, d_model=1024,
                              train=True, table_seed_=1003),
    "decode": Workload("decode", T=8, H=4, d_half=512, n_sub=4096, k=32, d_v=1024,
                       dtype="bf16", seed=1005, memplus=True, d_model=1024,
                       decode_steps=256, table_seed_=1003),
}

_DEVICE_GEN_BYTES = 64 << 20


def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _randn(shape, std: float, gen: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def value_table(w: Workload, device) -> torch.Tensor:
    """[N, d_v] value table, N(0, 0.02), in the workload dtype on ``device``."""
    device = torch.device(device)
    rows, d = w.N, w.d_v
    out = torch.empty(rows, d, dtype=w.torch_dtype, device=device)
    if device.type == "cpu" or rows * d * w.elem_bytes <= _DEVICE_GEN_BYTES:
        g = _cpu_gen(w.table_seed + 7)
        out.copy_(_randn((rows, d), 0.02, g))
        return out
    g = torch.Generator(device=device)
    g.manual_seed(w.table_seed + 7)
    chunk = max(1, (32 << 20) // d)  # 32 Mi elements per draw
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        tmp = torch.randn(r1 - r0, d, generator=g, device=device, dtype=torch.float32)
        out[r0:r1].copy_(tmp.mul_(0.02))
        del tmp
    return out


def value_shard(w: Workload, n_rows: int, rank: int, device) -> torch.Tensor:
    """[n_rows, d_v] rows N(0, 0.02) standing in for one rank's share of the
    value table in a row-sharded run: the same distribution as value_table,
    drawn from the rank's own stream (not the full table's values)."""
    out = torch.empty(max(0, n_rows), w.d_v, dtype=w.torch_dtype, device=device)
    g = torch.Generator(device=device)
    g.manual_seed(w.table_seed * 1000003 + 7 + rank)
    chunk = max(1, (32 << 20) // w.d_v)
    for r0 in range(0, n_rows, chunk):
        r1 = min(n_rows, r0 + chunk)
        tmp = torch.randn(r1 - r0, w.d_v, generator=g, device=device, dtype=torch.float32)
        out[r0:r1].copy_(tmp.mul_(0.02))
        del tmp
    return out


def _zipf_direction(w: Workload, g: torch.Generator) -> torch.Tensor:
    e = torch.randn(w.H, 2, w.d_half, generator=g, dtype=torch.float32)
    return e / e.norm(dim=-1, keepdim=True)


def make_inputs(w: Workload, device="cpu", with_values: bool = True) -> dict:
    """All inputs of one forward (and, for ``train``, backward) of ``w``.

    Each tensor family has its own generator stream, so the tables do not
    depend on T: the decode workload reuses the Memory+ tables exactly.
    """
    ts = w.table_seed
    dt = w.torch_dtype
    q = _randn((w.T, w.H, 2, w.d_half), 1.0, _cpu_gen(w.seed))
    gk = _cpu_gen(ts + 1)
    K = _randn((w.H, 2, w.n_sub, w.d_half), 1.0 / math.sqrt(w.d_half), gk)
    if w.zipf_beta > 0.0:
        e = _zipf_direction(w, gk)  # [H, 2, d_half]
        rank = torch.empty(w.H, 2, w.n_sub, dtype=torch.float32)
        for h in range(w.H):
            for c in range(2):
                perm = torch.randperm(w.n_sub, generator=gk)
                rank[h, c, perm] = torch.arange(w.n_sub, dtype=torch.float32)
        amp = w.zipf_beta * (rank + 1.0).pow(-w.zipf_alpha)  # [H,2,n]
        K = K + amp.unsqueeze(-1) * e.unsqueeze(2)
        q = q + w.zipf_gamma * e.unsqueeze(0)
    out = dict(query=q.to(dt).to(device), subkeys=K.to(dt).to(device))
    if w.memplus:
        out["x"] = _randn((w.T, w.d_model), 1.0, _cpu_gen(w.seed + 2)).to(dt).to(device)
        gw = _cpu_gen(ts + 3)
        s = 1.0 / math.sqrt(1024.0)
        out["W1"] = _randn((w.d_model, w.d_v), s, gw).to(dt).to(device)
        out["W2"] = _randn((w.d_v, w.d_model), s, gw).to(dt).to(device)
    if w.train:
        out["dy"] = _randn((w.T, w.d_out), 1.0, _cpu_gen(w.seed + 4)).to(dt).to(device)
    if with_values:
        out["values"] = value_table(w, device)
    return out


def decode_step_inputs(w: Workload, step: int, device="cpu") -> dict:
    """Fresh queries (and gate inputs) of decode step ``step``."""
    g = _cpu_gen(w.seed * 100003 + step)
    dt = w.torch_dtype
    out = dict(query=_randn((w.T, w.H, 2, w.d_half), 1.0, g).to(dt).to(device))
    if w.memplus:
        out["x"] = _randn((w.T, w.d_model), 1.0, g).to(dt).to(device)
    return out


def random_bags(n_bags: int, B: int, n_rows: int, seed: int,
                zipf: Optional[float] = None):
    """Row ids int32 [n_bags, B] and weights fp32 [n_bags, B] for testing the
    generic bag gather.  Weights are positive and sum to 1 per bag."""
    g = _cpu_gen(seed)
    if zipf is None:
        idx = torch.randint(0, n_rows, (n_bags, B), generator=g, dtype=torch.int64)
    else:
        ranks = torch.arange(1, n_rows + 1, dtype=torch.float64)
        p = ranks.pow(-zipf)
        idx = torch.multinomial((p / p.sum()).float(), n_bags * B, replacement=True,
                                generator=g).view(n_bags, B)
    wt = torch.rand(n_bags, B, generator=g, dtype=torch.float32) + 0.05
    wt = wt / wt.sum(dim=1, keepdim=True)
    return idx.to(torch.int32), wt


# ------------------------------------------------------------ Engram --

@dataclasses.dataclass(frozen=True)
class EngramWorkload:
    name: str
    n_seq: int
    L: int
    orders: tuple
    K: int
    rows_per_head: tuple
    d: int
    dtype: str = "bf16"
    vocab: int = 1 << 17
    seed: int = 2001        # tokens and hidden state
    table_seed: int = 2003  # the stacked table and the hash seeds

    @property
    def T(self) -> int:
        return self.n_seq * self.L

    @property
    def heads(self) -> int:
        return len(self.orders) * self.K

    @property
    def n_rows(self) -> int:
        return int(sum(self.rows_per_head))

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    @property
    def elem_bytes(self) -> int:
        return 2 if self.dtype == "bf16" else 4

    @property
    def seeds(self) -> tuple:
        """One 64-bit hash seed per head, drawn from the workload seed."""
        g = _cpu_gen(self.table_seed + 1)
        return tuple(int(x) for x in torch.randint(0, 2 ** 62, (self.heads,), generator=g))

    def scaled(self, **kw) -> "EngramWorkload":
        return dataclasses.replace(self, **kw)

    def describe(self) -> dict:
        return dict(workload=self.name, n_seq=self.n_seq, L=self.L, tokens=self.T,
                    orders=list(self.orders), hashes_per_order=self.K, d=self.d,
                    table_rows=self.n_rows, dtype=self.dtype)


ENGRAM = EngramWorkload("engram", n_seq=8, L=2048, orders=(2, 3), K=4,
                        rows_per_head=(1048573, 1048571, 1048559, 1048549, 1048517, 1048507,
                                       1048447, 1048433), d=1024)


def make_engram_inputs(w: EngramWorkload, device="cpu") -> dict:
    """tokens int32 [n_seq, L] uniform over the vocabulary, the stacked
    table [n_rows, d] N(0, 0.02) and the hidden state h [T, d] N(0, 1)."""
    device = torch.device(device)
    tok = torch.randint(0, w.vocab, (w.n_seq, w.L), generator=_cpu_gen(w.seed),
                        dtype=torch.int64).to(torch.int32)
    h = _randn((w.T, w.d), 1.0, _cpu_gen(w.seed + 1)).to(w.torch_dtype)
    table = torch.empty(w.n_rows, w.d, dtype=w.torch_dtype, device=device)
    if device.type == "cpu" or w.n_rows * w.d * w.elem_bytes <= _DEVICE_GEN_BYTES:
        table.copy_(_randn((w.n_rows, w.d), 0.02, _cpu_gen(w.table_seed + 7)))
    else:
        g = torch.Generator(device=device)
        g.manual_seed(w.table_seed + 7)
        chunk = max(1, (32 << 20) // w.d)
        for r0 in range(0, w.n_rows, chunk):
            r1 = min(w.n_rows, r0 + chunk)
            tmp = torch.randn(r1 - r0, w.d, generator=g, device=device, dtype=torch.float32)
            table[r0:r1].copy_(tmp.mul_(0.02))
            del tmp
    return dict(tokens=tok.to(device), table=table, h=h.to(device))
