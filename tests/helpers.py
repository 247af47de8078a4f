"""Shared helpers of the GPU parity tests: oracle inputs from the generator and
the acceptance check (relative L2 <= 1e-5 and |y - y_oracle| <= 1e-4 * m
element-wise, m = sum |w| |x| of the accumulation)."""
import numpy as np

import oracle
import synth

REL_L2 = 1e-5
ELEM = 1e-4


def mat(spec: synth.MatrixSpec) -> oracle.Mat:
    return oracle.Mat(spec.bits, spec.codes(), spec.scales())


def check_close(y, ref, mag, rel_l2=REL_L2, elem=ELEM, what=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    mag = np.asarray(mag, dtype=np.float64)
    assert y.shape == ref.shape, (y.shape, ref.shape)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    num = np.linalg.norm(y - ref)
    den = np.linalg.norm(ref)
    rel = num / den if den > 0 else num
    err = np.abs(y - ref)
    bound = elem * mag + 1e-30
    worst = float(np.max(err / bound))
    assert rel <= rel_l2, f"{what}: rel L2 {rel:.3e} > {rel_l2}"
    assert worst <= 1.0, f"{what}: element error {worst:.3f} x the 1e-4*m bound"
    return rel, worst


class OracleLayer:
    """Oracle view of a SynthLayer: raw codes/scales regenerated on the host."""

    def __init__(self, layer):
        self.layer = layer
        self._cache = {}

    def _m(self, kind, e):
        key = (kind, e)
        if key not in self._cache:
            self._cache[key] = mat(self.layer.spec(kind, e))
        return self._cache[key]

    def expert(self, e):
        return tuple(self._m(k, e) for k in (synth.KIND_GATE, synth.KIND_UP, synth.KIND_DOWN))

    def shared(self):
        if not self.layer.has_shared:
            return None
        return tuple(self._m(k, 0) for k in (synth.KIND_SH_GATE, synth.KIND_SH_UP, synth.KIND_SH_DOWN))

    def token(self, x_f64, idx_row, w_row, bf16_ops=False):
        return oracle.moe_token([self.expert(int(e)) for e in idx_row], w_row, self.shared(), x_f64, bf16_ops)
