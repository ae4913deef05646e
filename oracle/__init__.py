"""Oracle for the Sketch&Walk hot path: plain, slow, fp64, CPU only.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import or call anything in this package. The
product path (the CUDA library and its Python binding) never does, and this
package imports nothing from it.

Every function states the passage of "Scout Before You Attend: Sketch-and-Walk
Sparse Attention for Efficient LLM Inference" (the blog deep-dive on the paper,
arXiv 2602.07397) that it follows, by section and equation.
"""
from .sws_oracle import *  # noqa: F401,F403
