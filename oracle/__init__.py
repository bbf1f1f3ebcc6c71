"""CPU oracle for the VC-Attention forward path.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (``bit_fp8_attention_prep_b200``) never imports it and
shares no code with it.

``vc_oracle`` (numpy, fp64) is the oracle; ``ref_cpp`` loads a second statement
of its main path in plain C++ (``vc_oracle_ref.cpp``), held against it bit for bit
by the tests.
"""
from .vc_oracle import *  # noqa: F401,F403
