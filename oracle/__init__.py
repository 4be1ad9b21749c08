"""Oracle for the Muon step: plain fp64 numpy, test infrastructure only.

Importable by the tests, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py``; never by the library itself.  See ``oracle.muon`` for what it
computes and the readings it takes where the documentation is silent.
"""
from . import muon, emulate  # noqa: F401
from .muon import (DEFAULT_COEFFS, NORM_EPS, apply_update, assign_owners, clip_grad_norm,  # noqa: F401
                   clip_grad_norm_buckets,
                   coeff_schedule, ns_iteration_flops,
                   frobenius_normalize, gram_ns_iterations, lr_scale, momentum_update,
                   muon_step, newton_schulz, orient, shape_groups)
