"""Torch-facing wrapper of the C ABI: owns the device tensors (Pi, S,
workspace, outputs) and forwards every call to libtq.  Inputs given on the
host are copied to the device first; all arithmetic runs in libtq's kernels.
"""
from dataclasses import dataclass

import torch

from . import _binding as B


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _dtype_code(t):
    if t.dtype == torch.float32:
        return B.TQ_F32
    if t.dtype == torch.bfloat16:
        return B.TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ptr(t):
    return t.data_ptr() if t is not None else None


@dataclass
class Codes:
    """Packed records: codes [G, n, b*d/32] int32 (bit pattern of uint32),
    xnorm, rnorm [G, n] float32."""
    codes: torch.Tensor
    xnorm: torch.Tensor
    rnorm: torch.Tensor

    @property
    def n(self):
        return self.codes.shape[1]


class Workspace:
    """Grow-only device scratch buffer for libtq calls."""

    def __init__(self, device):
        self.device = device
        self.buf = torch.empty(0, dtype=torch.uint8, device=device)

    def get(self, nbytes):
        if nbytes == (1 << 64) - 1:
            raise B.TQError("tq_workspace_bytes", B.TQ_ERR_UNSUPPORTED)
        if self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf.data_ptr(), self.buf.numel()


class TurboQuant:
    """TurboQuant quantizer with b total bits per coordinate for dimension d and
    G groups (KV heads), each group with its own Pi (and S) from seed + g.

    variant="prod" (default): the inner-product quantizer, (b-1)-bit
    Lloyd-Max index + 1 QJL sign bit, unbiased inner products.
    variant="mse": the MSE-only quantizer, b-bit Lloyd-Max index, no QJL
    (no S; biased inner products).
    A fractional b (1.5, 2.5, 3.5; inner-product quantizer only) gives the
    first d/2 rotated coordinates ceil(b) bits and the rest floor(b)
    (tq_build_codebook_split); self.b is then ceil(b) and self.split True."""

    def __init__(self, d, b, seed=0, groups=1, device="cuda", variant="prod"):
        if variant not in ("prod", "mse"):
            raise ValueError(f"variant must be 'prod' or 'mse', got {variant!r}")
        self.split = float(b) != int(b)
        if self.split and (variant != "prod" or float(b) * 2 != int(float(b) * 2)):
            raise ValueError(f"fractional widths are b - 1/2 of the inner-product quantizer, "
                             f"got b={b!r}, variant={variant!r}")
        self.d, self.seed, self.G = int(d), int(seed), int(groups)
        self.b = int(float(b) + 0.5) if self.split else int(b)
        self.variant = variant
        self.device = torch.device(device)
        self.Pi = torch.empty(self.G, d, d, dtype=torch.float32, device=self.device)
        self.S = (torch.empty(self.G, d, d, dtype=torch.float32, device=self.device)
                  if variant == "prod" else None)
        self.cb = B.tq_codebook_t()
        self.ws = Workspace(self.device)
        nbytes = B.tq_workspace_bytes(B.TQ_OP_BUILD, d, self.b, self.G, 0, 0, 0)
        wp, wn = self.ws.get(nbytes)
        if self.split:
            B.tq_build_codebook_split(self.d, self.b, self.seed, self.G, self.cb, _ptr(self.Pi),
                                      _ptr(self.S), wp, wn, _stream())
        elif variant == "prod":
            B.tq_build_codebook(self.d, self.b, self.seed, self.G, self.cb, _ptr(self.Pi),
                                _ptr(self.S), wp, wn, _stream())
        else:
            B.tq_build_codebook_mse(self.d, self.b, self.seed, self.G, self.cb, _ptr(self.Pi),
                                    wp, wn, _stream())

    @property
    def words(self):
        if self.split:
            return self.d // 64 * (2 * self.b - 1)
        return self.b * self.d // 32

    def centroids(self):
        return torch.tensor(list(self.cb.centroids)[: self.cb.levels], dtype=torch.float32)

    def boundaries(self):
        return torch.tensor(list(self.cb.boundaries)[: max(self.cb.levels - 1, 0)],
                            dtype=torch.float32)

    def _grouped(self, x):
        if x.dim() == 2:
            x = x.unsqueeze(0)
        if x.dim() != 3 or x.shape[0] != self.G or x.shape[2] != self.d:
            raise ValueError(f"expected [G={self.G}, n, d={self.d}], got {tuple(x.shape)}")
        if x.device != self.device:
            x = x.to(self.device, non_blocking=True)
        return x.contiguous()

    def encode(self, x, out=None):
        x = self._grouped(x)
        n = x.shape[1]
        if out is None:
            out = Codes(torch.empty(self.G, n, self.words, dtype=torch.int32, device=self.device),
                        torch.empty(self.G, n, dtype=torch.float32, device=self.device),
                        torch.empty(self.G, n, dtype=torch.float32, device=self.device))
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_ENCODE, self.d, self.b, self.G, n, 0, 0))
        B.tq_encode(self.cb, _ptr(self.Pi), _ptr(self.S), self.G, n, _ptr(x), _dtype_code(x),
                    _ptr(out.codes), _ptr(out.xnorm), _ptr(out.rnorm), wp, wn, _stream())
        return out

    def score(self, codes, q, out=None):
        q = self._grouped(q)
        nq = q.shape[1]
        n = codes.n
        if out is None:
            out = torch.empty(self.G, nq, n, dtype=torch.float32, device=self.device)
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_SCORE, self.d, self.b, self.G, n, nq, 0))
        B.tq_score(self.cb, _ptr(self.Pi), _ptr(self.S), self.G, n, _ptr(codes.codes),
                   _ptr(codes.xnorm), _ptr(codes.rnorm), nq, _ptr(q), _dtype_code(q), _ptr(out),
                   wp, wn, _stream())
        return out

    def topk(self, codes, q, k, out=None):
        q = self._grouped(q)
        nq = q.shape[1]
        n = codes.n
        if out is None:
            out = (torch.empty(self.G, nq, k, dtype=torch.float32, device=self.device),
                   torch.empty(self.G, nq, k, dtype=torch.int64, device=self.device))
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_TOPK, self.d, self.b, self.G, n, nq, k))
        B.tq_topk(self.cb, _ptr(self.Pi), _ptr(self.S), self.G, n, _ptr(codes.codes),
                  _ptr(codes.xnorm), _ptr(codes.rnorm), nq, _ptr(q), _dtype_code(q), k,
                  _ptr(out[0]), _ptr(out[1]), wp, wn, _stream())
        return out

    def attention_decode(self, kcodes, values, vcodes, q, scale=None, out=None):
        """Softmax attention of the queries q [G, nq, d] over the keys encoded
        by this (inner-product) quantizer and the values encoded by `values`
        (an MSE-only TurboQuant of the same d and groups): [G, nq, d] fp32.
        scale defaults to 1/sqrt(d)."""
        q = self._grouped(q)
        nq = q.shape[1]
        n = kcodes.n
        if scale is None:
            scale = self.d ** -0.5
        if out is None:
            out = torch.empty(self.G, nq, self.d, dtype=torch.float32, device=self.device)
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_ATTENTION, self.d, self.b, self.G, n,
                                                  nq, 0))
        B.tq_attention_decode(self.cb, _ptr(self.Pi), _ptr(self.S), values.cb, _ptr(values.Pi),
                              self.G, n, _ptr(kcodes.codes), _ptr(kcodes.xnorm),
                              _ptr(kcodes.rnorm), _ptr(vcodes.codes), _ptr(vcodes.xnorm), nq,
                              _ptr(q), _dtype_code(q), float(scale), _ptr(out), wp, wn, _stream())
        return out

    def score_topk(self, codes, q, k, scores_out=None, topk_out=None):
        """score() and topk() from one scoring pass: (scores [G, nq, n],
        (vals, ids) [G, nq, k])."""
        q = self._grouped(q)
        nq = q.shape[1]
        n = codes.n
        if scores_out is None:
            scores_out = torch.empty(self.G, nq, n, dtype=torch.float32, device=self.device)
        if topk_out is None:
            topk_out = (torch.empty(self.G, nq, k, dtype=torch.float32, device=self.device),
                        torch.empty(self.G, nq, k, dtype=torch.int64, device=self.device))
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_SCORE_TOPK, self.d, self.b, self.G, n,
                                                  nq, k))
        B.tq_score_topk(self.cb, _ptr(self.Pi), _ptr(self.S), self.G, n, _ptr(codes.codes),
                        _ptr(codes.xnorm), _ptr(codes.rnorm), nq, _ptr(q), _dtype_code(q), k,
                        _ptr(scores_out), _ptr(topk_out[0]), _ptr(topk_out[1]), wp, wn, _stream())
        return scores_out, topk_out

    def decode(self, codes, out=None):
        n = codes.n
        if out is None:
            out = torch.empty(self.G, n, self.d, dtype=torch.float32, device=self.device)
        wp, wn = self.ws.get(B.tq_workspace_bytes(B.TQ_OP_DECODE, self.d, self.b, self.G, n, 0, 0))
        B.tq_decode(self.cb, _ptr(self.Pi), _ptr(self.S), self.G, n, _ptr(codes.codes),
                    _ptr(codes.xnorm), _ptr(codes.rnorm), _ptr(out), wp, wn, _stream())
        return out


def logits_fp32(keys, q, out=None):
    """Exact fp32 logits <q, k> for keys [G, n, d] fp32 and queries [G, nq, d]."""
    G, n, d = keys.shape
    nq = q.shape[1]
    if out is None:
        out = torch.empty(G, nq, n, dtype=torch.float32, device=keys.device)
    B.tq_logits_fp32(d, G, n, _ptr(keys), nq, _ptr(q), _dtype_code(q), _ptr(out), _stream())
    return out


def exact_topk(x, q, k, ws=None):
    """Exact fp32 inner-product top-k: x [G, n, d] fp32, q [G, nq, d]."""
    G, n, d = x.shape
    nq = q.shape[1]
    vals = torch.empty(G, nq, k, dtype=torch.float32, device=x.device)
    ids = torch.empty(G, nq, k, dtype=torch.int64, device=x.device)
    ws = ws or Workspace(x.device)
    wp, wn = ws.get(B.tq_workspace_bytes(B.TQ_OP_EXACT, d, 1, G, n, nq, k))
    B.tq_exact_topk(d, G, n, _ptr(x), nq, _ptr(q), _dtype_code(q), k, _ptr(vals), _ptr(ids), wp,
                    wn, _stream())
    return vals, ids
