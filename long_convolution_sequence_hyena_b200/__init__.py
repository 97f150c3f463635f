"""Hyena operator (order-N gated FFT long convolution) for NVIDIA B200, sm_100a.

* ``capi``      -- ctypes binding of the C ABI in ``include/hyena.h`` (libhyena.so)
* ``api``       -- ``Plan``: torch tensors in, the same C calls underneath
* ``workloads`` -- seeded synthetic inputs (no operator arithmetic)
* ``build``     -- compiles ``csrc/*.cu`` into ``libhyena.so`` for sm_100a

Importing the package does not load the CUDA library; ``capi`` (and ``api``)
load it on import and raise if it is missing.
"""


def __getattr__(name):
    if name in ("Plan", "HyenaError"):
        from . import api
        return getattr(api, name)
    raise AttributeError(name)
