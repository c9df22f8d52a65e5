"""rlscan: RL credit assignment as one first-order linear-recurrence scan,
on hand-written CUDA kernels for B200 (sm_100a).

The compute entry points live in the C-ABI library ``librlscan.so``
(declared in ``include/rlscan.h``); ``rlscan`` is the thin ctypes binding
with the same names plus ``compute_*`` conveniences that allocate outputs.
The binding loads lazily so that ``workloads`` (seeded inputs) imports
without the library; every compute call goes to the CUDA library and fails
loudly when the library is missing or no CUDA device is present.
"""


def __getattr__(name):
    if name.startswith(("rlscan_", "compute_")) or name in ("RlscanError", "library_path"):
        from . import rlscan as _binding
        return getattr(_binding, name)
    raise AttributeError(name)
