"""Plain fp64 CPU oracle for the QJL key sketch, value quantizer and decode attention.

This package is TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py`` (its ``cpu_baseline`` leg and its ``--impl reference`` arm) may
import it. The CUDA library and its Python binding never import, link or call
anything here, and nothing here imports the library: the two share no code.

Every function restates what the method computes, citing the page that defines
it. The pages are:
  * "QJL: 1-Bit Quantized JL Transform for KV Cache Quantization with Zero
    Overhead" (atlas.scime.ai summary): sections Approach, Surprising findings
    and Limitations. This is the only page that describes the method.
  * "2 numbers out of 128 destroy the entire KV cache" (Towards AI): sections
    "The Obvious Fix: Use Fewer Bits" and "Why Outliers Destroy Quantization"
    (min-max quantization, outlier channels).
  * "Your Brain Already Runs on 1-Bit Keys" (0x01.fyi): sections "How Attention
    Computes a Score" and "Why Truncation Kills" (dot product, softmax).
  * TurboQuant slides, section 05 "Why Compressing the KV Cache Is Hard".

Parity status of each function is listed in ``qjl_oracle.PIN_STATUS``. Every
function there is pinned by a ``-m "not gpu"`` test; none is "parity unpinned".
"""

from .qjl_oracle import *  # noqa: F401,F403
