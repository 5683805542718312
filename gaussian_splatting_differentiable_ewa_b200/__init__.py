"""B200-native differentiable EWA Gaussian splatting (sm_100a CUDA + C-ABI).

The compute path lives in ``libgs_b200.so`` (``csrc/``); ``api`` is the thin
ctypes binding with the same call names. ``scenes`` draws seeded synthetic
inputs. Importing this package loads nothing; the library is loaded on first
use of ``api``.
"""

__all__ = ["api", "scenes"]


def __getattr__(name):
    if name in ("api", "scenes"):
        import importlib
        return importlib.import_module(__name__ + "." + name)
    raise AttributeError(name)
