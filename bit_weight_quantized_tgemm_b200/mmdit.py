"""The ternary linears of one MMDiT denoising step, run back to back from a CUDA graph.

Block structure: 5 joint blocks and 20 single blocks, 24 heads
("We're Teaching Your Browser to Paint", "Then we ported in layers"). Widths are hidden
3072 and MLP 12288, the shapes of the step's matmuls. Each block's linears are:

* joint block, once per stream (image tokens, text tokens), each stream with its own
  weights: qkv 9216x3072, attention out 3072x3072, MLP up 12288x3072, MLP down
  3072x12288;
* single block (image and text tokens together):
  - ``linear1``: the qkv and MLP-up rows stacked into one packed 21504x3072 matrix; its
    qkv and MLP parts are row ranges of that matrix, i.e. pointer offsets ("Slice
    weights, not activations");
  - ``linear2``: the fused out projection y = attn W1^T + mlp W2^T (K1 = 3072,
    K2 = 12288), split along its input axis into one two-input call.

Before the blocks, the text tokens' 7,680-wide conditioning is projected to 3072
(``context``), with the width from "You Can Now Just Ask for an Image", "Closing the last
gap: the text encoder". That makes
81 linears on the token path, out of the model's 100 big matrices ("mindview-t2i-turbo",
"One step"). The modulation and time-embedding layers act on one vector per step, and
that vector depends only on the step. They are computed ahead of time (same section),
so they are not part of this sequence.

Attention, norms, RoPE and the MLP activation are out of scope. Each linear reads a
synthetic activation buffer of its shape, so the sequence measures the matmul share of
a step. Weights are seeded synthetic Q2_0 data packed on the device: codes uniform in
{0, 1, 2}, block scales |N(0, 0.02)| rounded to f16. The packed bytes differ per linear
and total about 0.9 GB, which is more than L2 holds, so a replay streams them from HBM.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Optional, Tuple

import torch

from . import binding as tg

HIDDEN = 3072
MLP = 12288
QKV = 3 * HIDDEN
COND = 7680  # text conditioning width: three 2560-wide reader layers


@dataclass
class Linear:
    """One matmul of the sequence.

    y[M][N] = x[M][K] . W^T (+ x2[M][K2] . W2^T when K2 > 0). The weight is rows
    [row0, row0 + N) of the packed matrix `weight` (and of `weight2`)."""
    name: str
    M: int
    N: int
    K: int
    weight: str
    row0: int = 0
    K2: int = 0
    weight2: str = ""

    @property
    def flops(self) -> int:
        return 2 * self.M * self.N * (self.K + self.K2)


def step_linears(img_tokens: int = 1024, txt_tokens: int = 512, joint_blocks: int = 5,
                 single_blocks: int = 20, slice_rows: bool = False) -> List[Linear]:
    """The token-path linears of one step, in execution order.

    slice_rows: run a single block's linear1 as two calls on the qkv and MLP-up row
    ranges of its packed matrix, instead of one call over all 21504 rows."""
    seq: List[Linear] = [Linear("context", txt_tokens, HIDDEN, COND, "context")]
    for b in range(joint_blocks):
        for stream, m in (("img", img_tokens), ("txt", txt_tokens)):
            p = f"joint{b}.{stream}"
            seq += [Linear(f"{p}.qkv", m, QKV, HIDDEN, f"{p}.qkv"),
                    Linear(f"{p}.out", m, HIDDEN, HIDDEN, f"{p}.out"),
                    Linear(f"{p}.mlp_up", m, MLP, HIDDEN, f"{p}.mlp_up"),
                    Linear(f"{p}.mlp_down", m, HIDDEN, MLP, f"{p}.mlp_down")]
    m = img_tokens + txt_tokens
    for b in range(single_blocks):
        p = f"single{b}"
        if slice_rows:
            seq += [Linear(f"{p}.linear1.qkv", m, QKV, HIDDEN, f"{p}.linear1", 0),
                    Linear(f"{p}.linear1.mlp_up", m, MLP, HIDDEN, f"{p}.linear1", QKV)]
        else:
            seq.append(Linear(f"{p}.linear1", m, QKV + MLP, HIDDEN, f"{p}.linear1"))
        seq.append(Linear(f"{p}.linear2", m, HIDDEN, HIDDEN, f"{p}.linear2.attn", 0, MLP,
                          f"{p}.linear2.mlp"))
    return seq


def weight_shapes(joint_blocks: int = 5, single_blocks: int = 20) -> Dict[str, Tuple[int, int]]:
    """Packed matrices (rows, K) by name."""
    shapes: Dict[str, Tuple[int, int]] = {"context": (HIDDEN, COND)}
    for b in range(joint_blocks):
        for stream in ("img", "txt"):
            p = f"joint{b}.{stream}"
            shapes[f"{p}.qkv"] = (QKV, HIDDEN)
            shapes[f"{p}.out"] = (HIDDEN, HIDDEN)
            shapes[f"{p}.mlp_up"] = (MLP, HIDDEN)
            shapes[f"{p}.mlp_down"] = (HIDDEN, MLP)
    for b in range(single_blocks):
        p = f"single{b}"
        shapes[f"{p}.linear1"] = (QKV + MLP, HIDDEN)
        shapes[f"{p}.linear2.attn"] = (HIDDEN, HIDDEN)
        shapes[f"{p}.linear2.mlp"] = (HIDDEN, MLP)
    return shapes


def make_weights(shapes: Dict[str, Tuple[int, int]], seed: int = 0,
                 device: str = "cuda") -> Dict[str, Tuple[torch.Tensor, torch.Tensor]]:
    """Seeded synthetic ternary matrices packed on the device: name -> (wq, d)."""
    g = torch.Generator(device=device).manual_seed(seed)
    out = {}
    for name in sorted(shapes):
        n, k = shapes[name]
        codes = torch.randint(0, 3, (n, k), dtype=torch.uint8, device=device, generator=g)
        scale = (torch.randn(n, k // 128, device=device, generator=g).abs() * 0.02).half().float()
        wq, d, status = tg.q2_pack(codes, scale)
        if int(status.item()) != 0:
            raise RuntimeError(f"packing {name} failed with status {int(status.item())}")
        out[name] = (wq, d)
        del codes, scale
    return out


@dataclass
class _Call:
    lin: Linear
    x: torch.Tensor
    x2: Optional[torch.Tensor]
    y: torch.Tensor
    wq: torch.Tensor
    d: torch.Tensor
    wq2: Optional[torch.Tensor] = None
    d2: Optional[torch.Tensor] = None


@dataclass
class StepSequence:
    """Buffers and calls for one step's linears; `run()` issues them on the current stream.

    Activations are one buffer per distinct (M, K) input shape and one per (M, N) output
    shape, shared by the layers of that shape, unless `distinct_outputs` gives every
    linear its own output (for checking each one). One workspace of the largest size any
    call asks for serves all calls, which run one after another on one stream."""
    linears: List[Linear]
    weights: Dict[str, Tuple[torch.Tensor, torch.Tensor]]
    out_dtype: int = tg.OUT_BF16
    distinct_outputs: bool = False
    seed: int = 1
    calls: List[_Call] = field(default_factory=list)
    workspace: Optional[torch.Tensor] = None
    inputs: Dict[Tuple[int, int], torch.Tensor] = field(default_factory=dict)

    def __post_init__(self):
        g = torch.Generator(device="cuda").manual_seed(self.seed)
        xs = self.inputs  # (M, K) -> the activation buffer every linear of that shape reads
        ys: Dict[Tuple[int, int], torch.Tensor] = {}
        ydt = torch.float32 if self.out_dtype == tg.OUT_F32 else torch.bfloat16

        def x_of(m, k):
            if (m, k) not in xs:
                xs[(m, k)] = torch.randn(m, k, device="cuda", generator=g).bfloat16()
            return xs[(m, k)]

        ws = 256
        for lin in self.linears:
            wq, d = self.weights[lin.weight]
            kq = lin.K // 4
            wq = wq[lin.row0:lin.row0 + lin.N]  # a row range is a pointer offset
            d = d[lin.row0:lin.row0 + lin.N]
            if self.distinct_outputs:
                y = torch.empty(lin.M, lin.N, device="cuda", dtype=ydt)
            else:
                y = ys.setdefault((lin.M, lin.N), torch.empty(lin.M, lin.N, device="cuda", dtype=ydt))
            assert wq.shape[1] == kq
            if lin.K2:
                wq2, d2 = self.weights[lin.weight2]
                wq2 = wq2[lin.row0:lin.row0 + lin.N]
                d2 = d2[lin.row0:lin.row0 + lin.N]
                call = _Call(lin, x_of(lin.M, lin.K), x_of(lin.M, lin.K2), y, wq, d, wq2, d2)
                ws = max(ws, tg.dual_workspace_size(lin.M, lin.N, lin.K, lin.K2))
            else:
                call = _Call(lin, x_of(lin.M, lin.K), None, y, wq, d)
                ws = max(ws, tg.workspace_size(tg.OP_Q2, lin.M, lin.N, lin.K))
            self.calls.append(call)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device="cuda")

    @property
    def flops(self) -> int:
        return sum(lin.flops for lin in self.linears)

    @property
    def weight_bytes(self) -> int:
        """Packed bytes read per step (codes and scales of every linear)."""
        total = 0
        for lin in self.linears:
            for k in (lin.K, lin.K2):
                if k:
                    total += lin.N * (k // 4 + (k // 128) * 2)
        return total

    def run(self):
        ws = self.workspace
        for c in self.calls:
            if c.x2 is not None:
                tg.gemm_q2_dual(c.x, c.wq, c.d, c.x2, c.wq2, c.d2, out_dtype=self.out_dtype,
                                y=c.y, workspace=ws)
            else:
                tg.gemm_q2(c.x, c.wq, c.d, out_dtype=self.out_dtype, y=c.y, workspace=ws)

    def capture(self, warmup: int = 1) -> torch.cuda.CUDAGraph:
        """Capture `run()` in a CUDA graph (after `warmup` eager runs, which also set the
        kernels' attributes once); replay it with `graph.replay()`."""
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            for _ in range(warmup):
                self.run()
        s.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            self.run()
        torch.cuda.current_stream().wait_stream(s)
        return graph
