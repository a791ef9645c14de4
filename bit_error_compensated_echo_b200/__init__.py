"""Echo -- error-compensated 4-bit tensor-parallel all-reduce -- on B200.

The product is the C-ABI library libecho_b200.so (include/echo.h), built
from csrc/ by ``python -m bit_error_compensated_echo_b200.build``.
``abi`` binds its entry points under the same names; ``EchoPlan`` wraps them
for torch tensors.  ``workloads`` holds the seeded input generators.
Accessing ``abi`` or ``EchoPlan`` loads the library and raises if it is
missing: there is no fallback implementation.
"""

__all__ = ["EchoPlan", "EchoError", "abi", "workloads"]


def __getattr__(name):
    if name in ("EchoPlan",):
        from .api import EchoPlan
        return EchoPlan
    if name == "EchoError":
        from .abi import EchoError
        return EchoError
    if name in ("abi", "workloads", "api", "build"):
        import importlib
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
