"""Plain fp64 CPU oracle of the VDN hybrid attention layer.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check in
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` may
import, call or execute anything in this package. The product path (the C-ABI
library and its Python binding) never touches it, and it shares no code with
that path: it neither imports nor is imported by the package
``softmax_attention_video_vdn_b200``.
"""
from .vdn_oracle import *  # noqa: F401,F403
from .fp8 import *  # noqa: F401,F403
from .vdn_backward import *  # noqa: F401,F403
