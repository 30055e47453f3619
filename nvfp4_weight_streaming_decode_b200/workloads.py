"""Synthetic decode-round workloads built on the C ABI.

A round (ignis README, "The decode round") is, per layer, the q/k/v
projection (one 3*hidden x hidden matrix: the three share their input), the
o projection, the fused gate/up projection with SiLU-multiply, and the down
projection, followed by the vocabulary head.  Weights and inputs are drawn
with ``synth`` on the device, packed with ``nvfp4_pack_check``, and wired
into descriptors for ``nvfp4_round_create``.  Each GEMM reads a fixed
per-layer input (the layer input x_l for q/k/v and gate/up, a stand-in
attention output a_l for o, and the H just produced for down); no value
flows from one layer to the next, so the numbers stay N(0,1)-scaled without
norms while the graph is still one serial chain of nodes.

torch is used here for device memory only.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import abi, synth

BYTES_PER_WEIGHT = 0.5 + 1.0 / 16.0   # one nibble plus a scale byte per 16


@dataclass
class Matrix:
    tensor_id: int
    N: int
    K: int
    wq: torch.Tensor
    ws: torch.Tensor
    exp: tuple

    @property
    def weight_bytes(self) -> int:
        return self.N * self.K // 2 + self.N * self.K // 16

    def canonical(self, device, workload_id):
        """Regenerate this matrix's canonical planes (same seed) on `device`."""
        return synth.torch_matrix(workload_id, self.tensor_id, self.N, self.K, device, self.exp)


def make_matrix(workload_id, tensor_id, N, K, device, exp=synth.EXP_UNIFORM_M4_2) -> Matrix:
    q, s = synth.torch_matrix(workload_id, tensor_id, N, K, device, exp)
    wq, ws = abi.pack(q, s)
    del q, s
    return Matrix(tensor_id, N, K, wq, ws, exp)


@dataclass
class SyntheticRound:
    device: torch.device
    layers: int
    hidden: int
    ffn: int
    vocab: int
    workload_id: int = 4
    gscale: float = synth.GSCALE
    mats: dict = field(default_factory=dict)
    bufs: dict = field(default_factory=dict)
    descs: list = field(default_factory=list)
    nodes: list = field(default_factory=list)   # (name, kind, input key, output key, matrix keys)

    @classmethod
    def build(cls, device, layers=64, hidden=5120, ffn=17408, vocab=151936, workload_id=4):
        r = cls(torch.device(device), layers, hidden, ffn, vocab, workload_id)
        r._build()
        return r

    def _act(self, tid, K):
        return synth.torch_activations(self.workload_id, tid, abi_max_m(), K, self.device)

    def _build(self):
        L, h, f, v, dev, wid = self.layers, self.hidden, self.ffn, self.vocab, self.device, self.workload_id
        M8 = abi_max_m()
        for l in range(L):
            base = 10 * l
            self.mats[f"qkv{l}"] = make_matrix(wid, base + 0, 3 * h, h, dev)
            self.mats[f"o{l}"] = make_matrix(wid, base + 1, h, h, dev)
            self.mats[f"gate{l}"] = make_matrix(wid, base + 2, f, h, dev)
            self.mats[f"up{l}"] = make_matrix(wid, base + 3, f, h, dev)
            self.mats[f"down{l}"] = make_matrix(wid, base + 4, h, f, dev)
            self.bufs[f"x{l}"] = self._act(2 * l, h)
            self.bufs[f"a{l}"] = self._act(2 * l + 1, h)
            self.bufs[f"yqkv{l}"] = torch.zeros((M8, 3 * h), dtype=torch.float32, device=dev)
            self.bufs[f"yo{l}"] = torch.zeros((M8, h), dtype=torch.float32, device=dev)
            self.bufs[f"H{l}"] = torch.zeros((M8, f), dtype=torch.bfloat16, device=dev)
            self.bufs[f"ydown{l}"] = torch.zeros((M8, h), dtype=torch.float32, device=dev)
        self.mats["head"] = make_matrix(wid, 100000, v, h, dev)
        self.bufs["xhead"] = self._act(100000, h)
        self.bufs["logits"] = torch.zeros((M8, v), dtype=torch.float32, device=dev)
        G, D = abi.NVFP4_DESC_GEMM, abi.NVFP4_DESC_GATEUP_SILU
        for l in range(L):
            self._node(f"qkv{l}", G, f"x{l}", f"yqkv{l}", [f"qkv{l}"])
            self._node(f"o{l}", G, f"a{l}", f"yo{l}", [f"o{l}"])
            self._node(f"gateup{l}", D, f"x{l}", f"H{l}", [f"gate{l}", f"up{l}"])
            self._node(f"down{l}", G, f"H{l}", f"ydown{l}", [f"down{l}"])
        self._node("head", G, "xhead", "logits", ["head"])

    def _node(self, name, kind, xin, out, mkeys):
        m0 = self.mats[mkeys[0]]
        m1 = self.mats[mkeys[1]] if len(mkeys) > 1 else None
        self.descs.append(abi.desc(kind, self.bufs[xin], m0.wq, m0.ws, self.gscale, self.bufs[out],
                                   m0.N, m0.K, m1.wq if m1 else None, m1.ws if m1 else None,
                                   self.gscale if m1 else 0.0))
        self.nodes.append((name, kind, xin, out, mkeys))

    @property
    def weight_bytes(self) -> int:
        return sum(m.weight_bytes for m in self.mats.values())

    def run_direct(self, M, stream=None):
        """The same chain as the graph, as direct C-ABI calls (no graph, no PDL)."""
        for (name, kind, xin, out, mkeys) in self.nodes:
            m0 = self.mats[mkeys[0]]
            X = self.bufs[xin][:M]
            if kind == abi.NVFP4_DESC_GEMM:
                abi.gemm_decode(X, m0.wq, m0.ws, self.gscale, m0.N, m0.K,
                                Y=self.bufs[out][:M], stream=stream)
            else:
                m1 = self.mats[mkeys[1]]
                abi.gemm_gateup_silu(X, m0.wq, m0.ws, self.gscale, m1.wq, m1.ws, self.gscale,
                                     m0.N, m0.K, H=self.bufs[out][:M], stream=stream)


def abi_max_m() -> int:
    return 8
