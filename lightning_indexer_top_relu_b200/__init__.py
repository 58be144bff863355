"""IndexCache sparse-attention layer stack for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libindexcache.so`` built from
``csrc/``; :mod:`.indexcache` is its thin ctypes binding (argument marshalling
only).  :mod:`.synth` draws the seeded synthetic inputs.  Importing this
package loads nothing; importing :mod:`.indexcache` loads the CUDA library
and fails loudly when it is missing.
"""
