"""Recent-token window beside the packed cache (oracle; test only).

"RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract: its K3V2
AIME result is stated for a cache without an fp16 recent-key buffer, which
names such a buffer as an option of the packed serving path: the most recent
tokens stay unquantized. The abstract gives no detail; readings adopted:

* The window holds the keys and the values of the R most recent tokens of a
  sequence exactly as they were appended (16-bit floats), unquantized.
* A token is quantized - with the layer's plan, exactly as it would be
  without a window - when it leaves the window, i.e. once R newer tokens
  follow it. Tokens leave in order, so after T appended tokens the packed
  cache holds tokens [0, T - w) and the window tokens [T - w, T), with
  w = min(R, T), whatever the sizes of the appends were.
* Decode attends over the dequantized packed tokens and the exact window
  tokens together: softmax attention over their concatenation.
* Placement: the window is a ring of R slots; token t sits in slot t mod R.
"""
from __future__ import annotations

import numpy as np

from . import attn


def split_point(n_tokens: int, R: int) -> int:
    """Number of packed (quantized) tokens after n_tokens appends."""
    return n_tokens - min(R, n_tokens)


def ring_slots(n_tokens: int, R: int):
    """(token, slot) of every window token after n_tokens appends."""
    return [(t, t % R) for t in range(split_point(n_tokens, R), n_tokens)]


def decode(q, khat_heads, vhat_heads, kwin_heads, vwin_heads) -> np.ndarray:
    """Decode output [Hq, d] for one sequence: per KV head, attention over the
    dequantized packed tokens followed by the exact window tokens."""
    k = [np.concatenate([np.asarray(a, np.float64), np.asarray(b, np.float64)])
         for a, b in zip(khat_heads, kwin_heads)]
    v = [np.concatenate([np.asarray(a, np.float64), np.asarray(b, np.float64)])
         for a, b in zip(vhat_heads, vwin_heads)]
    return attn.decode(q, k, v)
