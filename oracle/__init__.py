"""CPU oracle for Positional-LSH approximate ALiBi attention.

TEST INFRASTRUCTURE ONLY. Only tests/, the smoke check in __graft_entry__.py
and the CPU-baseline leg of bench.py may import this package. The library
under alibi_positional_lsh_b200/ never imports it, and it imports nothing
from there: the two share no code.

Everything here is plain float64 numpy (plus Python integers for the
counter-based generator), written for readability, not speed.

Source: "Positional LSH: Binary Block Matrix Approximation for Attention with
Linear Biases" (Wolfson & Wagner), as summarised on the three gist.science
explainer pages (nl, zh, ja) of arXiv 2605.09472. Citations below name the
page and the section of its technical summary.

Parity status of each function: see the per-function docstrings. Every
function is pinned by a test under tests/ that checks it against something
other than itself (a published test vector, a hand-derived worked example, a
closed form, a library routine on a special case, or a statistical law);
no function is parity unpinned.
"""
from .plsh_oracle import *  # noqa: F401,F403
