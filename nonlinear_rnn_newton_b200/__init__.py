"""B200-native ParaRNN Newton solve (ParaGRU / ParaLSTM) behind a C ABI.

The CUDA library ``libpararnn.so`` (built in-tree by ``build.py``) does all
the work; ``capi`` is its thin ctypes binding, with the same entry-point
names as ``include/pararnn.h``.  ``workloads`` draws the seeded synthetic
inputs and needs no library.

Binding names are resolved on first use; if the library is not built that
first use raises ImportError (there is no fallback).
"""
import importlib

__all__ = [
    "PararnnError",
    "pararnn_cell_adjoint",
    "pararnn_cell_adjoint_workspace_size",
    "pararnn_cell_compile_log",
    "pararnn_cell_compute_warps",
    "pararnn_cell_create",
    "pararnn_cell_destroy",
    "pararnn_cell_solve",
    "pararnn_cell_solve_async",
    "pararnn_cell_workspace_size",
    "pararnn_gru_adjoint",
    "pararnn_gru_adjoint_workspace_size",
    "pararnn_gru_segment_pass",
    "pararnn_gru_segment_fold",
    "pararnn_gru_segment_combine",
    "pararnn_gru_sequential",
    "pararnn_gru_solve",
    "pararnn_gru_solve_async",
    "pararnn_gru_solve_noalloc",
    "pararnn_gru_solve_noalloc_max_scratch",
    "pararnn_gru_step",
    "pararnn_gru_workspace_size",
    "pararnn_linear_scan",
    "pararnn_linear_scan_workspace_size",
    "pararnn_lstm_adjoint",
    "pararnn_lstm_adjoint_workspace_size",
    "pararnn_lstm_segment_pass",
    "pararnn_lstm_segment_fold",
    "pararnn_lstm_segment_combine",
    "pararnn_lstm_sequential",
    "pararnn_lstm_solve",
    "pararnn_lstm_solve_async",
    "pararnn_lstm_step",
    "pararnn_lstm_workspace_size",
    "pararnn_read_pass_times",
    "pararnn_segment_record_floats",
    "pararnn_result_to_device",
    "pararnn_gru_project_workspace_size",
    "pararnn_gru_project_solve",
    "pararnn_gru_project_solve_async",
    "pararnn_segment_fold_workspace_size",
    "pararnn_read_result",
    "pararnn_selftest_wait_timeout",
]


def __getattr__(name):
    if name in __all__ or name == "capi":
        capi = importlib.import_module(".capi", __name__)
        return capi if name == "capi" else getattr(capi, name)
    raise AttributeError(name)
