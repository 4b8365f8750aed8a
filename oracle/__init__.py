"""Plain CPU oracle of the SpectralQuant compressed-KV hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this
package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it. It shares no code, table or constant generator
with the CUDA library; both sides implement the method independently from
the pages that describe it:

* SpectralQuant README (Dynamis-Labs/spectralquant), sections "Overview",
  "Key Findings" and "Repository Structure" (calibration.py: eigenspectral
  calibration -- PCA, d_eff, kappa; spectral_rotation.py; nonuniform_quantization.py:
  Lloyd-Max codebooks; selective_qjl.py: QJL correction on the signal dims only).
* spectralquant tests/conftest.py (v1 branch), fixture
  ``pre_computed_calibration`` (uncentered second moment, eigh, descending
  order, participation-ratio d_eff, spectral gap).
* TurboQuant reference implementation README (scos-lab/turboquant),
  "Algorithm Correctness" distortion table (prior art; used as a pin).

Everything is float64 NumPy, written for a reader to check by eye against
those passages. Where the pages leave a step open, the module that
implements it states the reading it takes.

Modules
-------
codebook     Gaussian Lloyd-Max scalar quantizers, b = 1..8 bits.
rng          SplitMix64 + Box-Muller: the Gaussian stream of the QJL matrix.
calibration  second moment, eigenbasis, d_eff, kappa, scales, water-filling.
codec        rotate, quantize, QJL signs, bit packing, and the inverse.
attention    decode attention read straight from the packed cache.
record       the byte layout of one head's calibration record.
"""

__all__ = ["codebook", "rng", "calibration", "codec", "attention", "record"]
