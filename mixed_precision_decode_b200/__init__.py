"""B200 (sm_100a) library for the decode hot path of BitsMoE's spectral MoE
gate/up projection: packing into width-grouped bit planes, the shared
projection z = Phi^T x and the routed bit-plane expert forward, behind the C
ABI in include/bitsmoe.h (libbitsmoe.so, built from csrc/)."""
from . import bitsmoe  # noqa: F401
from .layer import PackedProjection, SpectralMoELayer  # noqa: F401
