"""B200-native (sm_100a) Prox two-stage sparse SwiGLU FFN for small-batch decode.

The compute path lives in the CUDA library ``libprox.so`` (built from
``csrc/``) behind the C ABI declared in ``include/prox.h``; ``prox`` is its thin
Python binding. ``synth`` draws the seeded synthetic inputs. Importing the
package loads nothing: the library is opened on first use and a missing or
unloadable library raises instead of falling back to anything else.
"""
