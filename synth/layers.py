"""Synthetic MoE layers resident in device memory.

Draws codes and scales with the device twin of the generator (bit-identical to
the host generator the oracle side uses) and packs them with the library's
device packer into one buffer per matrix kind, experts at a fixed stride.
Recipe (the workload shapes): routed gate/up ROCmFP2, routed down ROCmFP3,
shared expert ROCmFP4; codes uniform over the levels; scales 0.02*2^U(-1,1).
"""
from __future__ import annotations

import torch

import synth

ROUTED_KINDS = (synth.KIND_GATE, synth.KIND_UP, synth.KIND_DOWN)
SHARED_KINDS = (synth.KIND_SH_GATE, synth.KIND_SH_UP, synth.KIND_SH_DOWN)


def _align(n: int, a: int = 256) -> int:
    return (n + a - 1) // a * a


class SynthLayer:
    """Packed device buffers of one synthetic layer (seed, layer)."""

    def __init__(self, seed: int, layer: int, H: int, I: int, E: int, k: int, fmts=(2, 2, 3), shared_fmts=(4, 4, 4),
                 has_shared: bool = True, device="cuda", experts=None):
        import block_quantized_moe_rocmfpx_b200 as rfx
        self.seed, self.layer, self.H, self.I, self.E, self.k = seed, layer, H, I, E, k
        self.fmts, self.shared_fmts, self.has_shared = tuple(fmts), tuple(shared_fmts), has_shared
        shapes = ((I, H), (I, H), (H, I))
        self.strides = tuple(_align(rfx.rfx_packed_bytes(f, r, c)) for f, (r, c) in zip(fmts, shapes))
        self.bufs = [torch.empty(E * s, dtype=torch.uint8, device=device) for s in self.strides]
        cmax = max(H, I) * max(H, I)
        codes = torch.empty(cmax, dtype=torch.uint8, device=device)
        scales = torch.empty(cmax // 32 * 2, dtype=torch.uint8, device=device)
        todo = range(E) if experts is None else experts
        for e in todo:
            for kind, f, (r, c), buf, s in zip(ROUTED_KINDS, fmts, shapes, self.bufs, self.strides):
                self._gen(kind, e, f, r, c, codes, scales, buf[e * s:(e + 1) * s])
        self.shared = None
        if has_shared:
            self.shared = []
            for kind, f, (r, c) in zip(SHARED_KINDS, shared_fmts, shapes):
                buf = torch.empty(_align(rfx.rfx_packed_bytes(f, r, c)), dtype=torch.uint8, device=device)
                self._gen(kind, 0, f, r, c, codes, scales, buf)
                self.shared.append(buf)
        torch.cuda.synchronize()
        self.packed_bytes_per_expert = sum(rfx.rfx_packed_bytes(f, r, c) for f, (r, c) in zip(fmts, shapes))
        self.shared_bytes = sum(rfx.rfx_packed_bytes(f, r, c) for f, (r, c) in zip(shared_fmts, shapes)) \
            if has_shared else 0

    def _gen(self, kind, e, f, rows, cols, codes, scales, dst):
        import block_quantized_moe_rocmfpx_b200 as rfx
        spec = synth.MatrixSpec(self.seed, self.layer, kind, e, f, rows, cols)
        synth.codes_dev(spec.code_key, f, rows, cols, codes)
        synth.scales_dev(spec.scale_key, f, rows, cols, scales)
        rfx.rfx_pack_device(f, codes, scales, rows, cols, dst)

    def spec(self, kind: int, expert: int) -> synth.MatrixSpec:
        H, I = self.H, self.I
        routed = kind in ROUTED_KINDS
        idx = (ROUTED_KINDS if routed else SHARED_KINDS).index(kind)
        f = (self.fmts if routed else self.shared_fmts)[idx]
        r, c = ((I, H), (I, H), (H, I))[idx]
        return synth.MatrixSpec(self.seed, self.layer, kind, expert if routed else 0, f, r, c)

    def moe_layer(self, max_T: int = 8):
        import block_quantized_moe_rocmfpx_b200 as rfx
        return rfx.MoeLayer(self.H, self.I, self.E, self.k, self.fmts, *self.bufs, self.strides,
                            shared=self.shared, shared_fmts=self.shared_fmts, max_T=max_T)

    def union_bytes(self, experts) -> int:
        """Packed weight bytes one pass reads for the given union of routed experts."""
        return len(set(int(e) for e in experts)) * self.packed_bytes_per_expert + self.shared_bytes
