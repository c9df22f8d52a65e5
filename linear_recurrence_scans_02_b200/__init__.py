"""rlscan: RL credit assignment as one first-order linear-recurrence scan,
on hand-written CUDA kernels for B200 (sm_100a).

The compute entry points live in the C-ABI library ``librlscan.so``
(declared in ``include/rlscan.h``); ``rlscan`` is the thin ctypes binding
with the same names plus ``compute_*`` conveniences that allocate outputs.
The binding loads lazily so that ``workloads`` (seeded inputs) imports
without the library; any compute call fails loudly when the library is
missing or no CUDA device is present.
"""
_BINDING_NAMES = {
    "rlscan_gae", "rlscan_vtrace", "rlscan_retrace", "rlscan_lambda_returns",
    "rlscan_discounted_returns", "rlscan_eligibility_traces", "rlscan_episodic_prefix_sum",
    "rlscan_workspace_bytes", "rlscan_check", "RlscanError",
    "compute_gae", "compute_vtrace", "compute_retrace", "compute_lambda_returns",
    "compute_discounted_returns", "compute_eligibility_traces", "compute_episodic_prefix_sum",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import rlscan as _b
        return getattr(_b, name)
    raise AttributeError(name)
