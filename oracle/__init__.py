"""fp64 CPU oracle for AXELRAM decode attention, the LOOKAT product-quantized keys and the power-of-two
shift-accumulate key codec (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline / reference arm may import this package.  The
product path (kv_cache_quantized_b200) never imports it, and the two share no code.
"""
from .axelram import *  # noqa: F401,F403
from .axelram import __all__ as _axelram_all
from .lookat import *  # noqa: F401,F403
from .lookat import __all__ as _lookat_all
from .pot import *  # noqa: F401,F403
from .pot import __all__ as _pot_all

__all__ = list(_axelram_all) + list(_lookat_all) + list(_pot_all)
