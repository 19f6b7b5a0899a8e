"""TTT layer inner-loop forward on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libttt.so`` (hand-written CUDA for
sm_100a, declared in ``include/ttt.h``); :mod:`.ttt` is a thin ctypes binding
that only marshals arguments.  There is no CPU fallback: every call fails
loudly when the library or a CUDA device is missing.
"""
from .ttt import (TTTError, last_device_status, library, linear_decode_step, linear_forward,  # noqa: F401
                  mlp_forward, status_string, version)
