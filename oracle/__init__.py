"""CPU oracle for the affine-quantised MoE FFN layer (fp64, plain C).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm may import this package; the
product path never does.  See ``oracle.c`` for the definitions and their
sources.
"""
from .oracle import (  # noqa: F401
    OracleTensor,
    OracleLayer,
    build,
    lib_path,
    set_threads,
    get_threads,
    unpack,
    dequant_f32,
    qmv,
    qmv_f64,
    route,
    route_f32,
    expert_ffn,
    layer,
    rmsnorm,
)
