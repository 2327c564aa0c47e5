"""B200-native joint text+image DiT attention forward (sm_100a).

The compute path lives in the CUDA library ``_lib/libjattn.so`` built from
``csrc/``; :mod:`.binding` is a thin ctypes layer over its C-ABI (declared in
``include/jattn.h``).  The library is loaded on first use and a missing or
unloadable library raises immediately: there is no CPU fallback.

Modules: :mod:`.attention` (one call per attention setting on raw Q, K, V),
:mod:`.ulysses` (CFG x Ulysses sequence parallelism around the kernels),
:mod:`.schedule` (which denoising steps stay dense), :mod:`.inputs` (seeded
synthetic workloads), :mod:`.build` (the in-tree sm_100a build).
"""
