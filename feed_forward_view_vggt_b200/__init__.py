"""B200-native hot path of VGGT's alternating-attention trunk.

Frame attention, global attention and AVGGT's Subsampled Global Attention
(SGA) over bf16 Q/K/V laid out [N, L, H, d], as hand-written sm_100a CUDA
kernels behind a C ABI (``include/vggt_attn.h``).  ``attn`` is the thin
ctypes binding with the same names as the C entry points; ``synth`` draws
the seeded synthetic inputs.  The binding loads ``libvggt_attn.so`` on first
use and raises if it is missing: there is no CPU fallback.
"""

__all__ = ["attn", "synth"]


def __getattr__(name):
    if name in ("attn", "synth"):
        import importlib

        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
