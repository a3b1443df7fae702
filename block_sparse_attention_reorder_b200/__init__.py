"""Block-sparse attention over 3D-tiled video latent tokens, for B200 (sm_100a).

The compute path is the C-ABI library libbsattn.so (include/bsattn.h) built
from csrc/; `block_sparse_attention_reorder_b200.bsattn` is its Python
binding. Importing the binding fails loudly when the library is not built.
`datagen` draws the seeded synthetic inputs.
"""

__all__ = ["bsattn", "datagen", "build"]


def __getattr__(name):
    if name in __all__:
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
