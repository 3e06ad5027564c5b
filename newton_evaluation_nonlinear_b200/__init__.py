"""Parallel Newton evaluation of nonlinear sequences on one NVIDIA B200.

Given s0 and f_1..f_T, every state s_t = f_t(s_{t-1}) is computed by the
fixed-point iteration s <- s - J~^{-1} F(s) with the Jacobi, Picard, diagonal
quasi-Newton or full Newton approximation J~ (web article "并行牛顿方法：加速非
线性序列评估的计算革命", jsqmd.com news item 789890, §1.2 and §2.2), each
iteration a fused cell + Jacobian evaluation and a chunked parallel scan
(§2.1), all in sm_100a CUDA kernels behind the C ABI of ``include/pn.h``.

This package is the ctypes binding of that library; see :mod:`._binding`.
"""
from ._binding import (MODES, PN_CELL_EULER_TANH, PN_CELL_GRU, PN_CELL_TANH_RNN, PN_ERR_CUDA,  # noqa: F401
                       PN_ERR_INVALID, PN_ERR_NOMEM, PN_ERR_NONFINITE, PN_ERR_TIMEOUT, PN_JACOBI,
                       PN_MAX_D_DIAG, PN_MAX_D_NEWTON, PN_NEWTON, PN_NOT_CONVERGED, PN_OK,
                       PN_OPT_DEBUG_STALL_TICKET, PN_OPT_DEVICE_LOOP, PN_OPT_NEWTON_BAND, PN_OPT_RUN_LENGTH, PN_OPT_SMALL_SOLVE, PN_OPT_TENSOR_CORES,
                       PN_OPT_WAIT_TIMEOUT_NS,
                       PN_PICARD, PN_QUASI, PN_STORE_BF16, PN_STORE_F16, PN_STORE_F32,
                       SIGNATURES, STATUS_NAMES, LIB_PATH, PnError, Solver, lib,
                       pn_activation, pn_create, pn_destroy, pn_dim, pn_eval, pn_eval_host, pn_eval_host_many, pn_eval_static, pn_eval_windowed, pn_get_residual_history,
                       pn_get_mode_history, pn_get_stats, pn_last_error, pn_reset_stats, pn_set_adaptive,
                       pn_set_damping, pn_set_option, pn_set_storage, pn_set_stream,
                       pn_time_iterations, pn_version)

__version__ = "0.1.0"
