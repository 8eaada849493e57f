"""ctypes declarations of include/gs.h for libgs.so.

Loading fails loudly (ImportError) when libgs.so has not been built: there is
no fallback path.  Build it with
``python -m gaussian_splatting_differentiable_tile_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
# GS_LIBRARY names the library file beside this module: libgs.so, or the
# checked build libgs_check.so
LIB_PATH = os.path.join(HERE, os.environ.get("GS_LIBRARY", "libgs.so"))

GS_TILE = 16
GS_OK = 0
GS_ERR_INVALID_ARG = -1
GS_ERR_CAPACITY = -2
GS_ERR_TOO_LARGE = -3
GS_ERR_ALIGNMENT = -4
GS_ERR_CUDA = -5
GS_ERR_DEVICE_TIMEOUT = -6
GS_ERR_BOUNDS = -7
GS_FLAG_TIGHT_TILES = 1
GS_FLAG_ANTIALIASED = 2
GS_FLAG_STOP_INCLUSIVE = 4
GS_FLAG_CAP_0999 = 8
GS_FLAG_RADII_AXIS = 16
GS_FLAG_RADII_OPACITY = 32
GS_FLAG_DEPTH = 64
GS_BIN_AUTO = 0
GS_BIN_PER_TILE = 1
GS_BIN_GLOBAL = 2

c_float_p = ctypes.c_void_p  # device pointers travel as plain addresses


class GsCamera(ctypes.Structure):
    _fields_ = [
        ("viewmat", ctypes.c_float * 16),
        ("fx", ctypes.c_float), ("fy", ctypes.c_float), ("cx", ctypes.c_float), ("cy", ctypes.c_float),
        ("width", ctypes.c_int32), ("height", ctypes.c_int32),
        ("near_z", ctypes.c_float),
        ("bg", ctypes.c_float * 3),
        ("flags", ctypes.c_uint32),
    ]


class GsParams(ctypes.Structure):
    _fields_ = [("means", ctypes.c_void_p), ("log_scales", ctypes.c_void_p), ("quats", ctypes.c_void_p),
                ("opacity_logits", ctypes.c_void_p), ("colors", ctypes.c_void_p)]


class GsGrads(ctypes.Structure):
    _fields_ = [("means", ctypes.c_void_p), ("log_scales", ctypes.c_void_p), ("quats", ctypes.c_void_p),
                ("opacity_logits", ctypes.c_void_p), ("colors", ctypes.c_void_p)]


class GsProjected(ctypes.Structure):
    _fields_ = [("xy_opacity_depth", ctypes.c_void_p), ("conic_radius", ctypes.c_void_p),
                ("rgb", ctypes.c_void_p), ("rect", ctypes.c_void_p), ("count", ctypes.c_void_p)]


class GsBins(ctypes.Structure):
    _fields_ = [
        ("pair_tile", ctypes.c_void_p), ("pair_gid", ctypes.c_void_p), ("ranges", ctypes.c_void_p),
        ("n_pairs", ctypes.c_void_p), ("status", ctypes.c_void_p),
        ("max_pairs", ctypes.c_int64), ("max_n", ctypes.c_int64),
        ("max_tiles", ctypes.c_int32), ("strategy", ctypes.c_int32),
        ("scratch", ctypes.c_void_p), ("scratch_bytes", ctypes.c_size_t),
    ]


GsParamSet = GsGrads  # gs_param_set: writable arrays in the gs_params layout


class GsAdamConfig(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_float * 5), ("eps", ctypes.c_float), ("beta1", ctypes.c_double),
                ("beta2", ctypes.c_double)]


class GsTrainLane(ctypes.Structure):
    _fields_ = [("proj", GsProjected), ("bins", GsBins), ("image", ctypes.c_void_p), ("T_final", ctypes.c_void_p),
                ("last", ctypes.c_void_p), ("dL_dimage", ctypes.c_void_p), ("grad2d", ctypes.c_void_p),
                ("grads", GsGrads), ("stream", ctypes.c_void_p), ("done", ctypes.c_void_p)]


class GsProfileStat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", ctypes.c_int32), ("total_ms", ctypes.c_float)]


# name -> (restype, argtypes); every function declared in include/gs.h
PROTOTYPES = {
    "gs_projected_bytes": (ctypes.c_size_t, [ctypes.c_int64]),
    "gs_projected_carve": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(GsProjected)]),
    "gs_bins_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32]),
    "gs_bins_carve": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                     ctypes.c_int32, ctypes.POINTER(GsBins)]),
    "gs_project": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsParams),
                                  ctypes.POINTER(GsProjected), ctypes.c_void_p]),
    "gs_bin_and_sort": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsProjected),
                                       ctypes.POINTER(GsBins), ctypes.POINTER(ctypes.c_int64),
                                       ctypes.c_void_p]),
    "gs_bin_and_sort_static": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64,
                                              ctypes.POINTER(GsProjected), ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64),
                                              ctypes.c_void_p]),
    "gs_render_fwd": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsProjected),
                                     ctypes.POINTER(GsBins), ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p]),
    "gs_render_fwd_l1": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsProjected),
                                        ctypes.POINTER(GsBins), ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]),
    "gs_render_bwd": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsParams),
                                     ctypes.POINTER(GsProjected), ctypes.POINTER(GsBins), ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.POINTER(GsGrads), ctypes.c_void_p]),
    "gs_render_features_fwd": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsProjected),
                                              ctypes.POINTER(GsBins), ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "gs_render_features_bwd": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsParams),
                                              ctypes.POINTER(GsProjected), ctypes.POINTER(GsBins), ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(GsGrads),
                                              ctypes.c_void_p]),
    "gs_render_stats": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int64, ctypes.POINTER(GsProjected),
                                       ctypes.POINTER(GsBins), ctypes.c_void_p, ctypes.c_void_p,
                                       ctypes.c_void_p]),
    "gs_l1_loss_grad": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                       ctypes.c_void_p, ctypes.c_void_p]),
    "gs_adam_step": (ctypes.c_int, [ctypes.c_int64, ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads), ctypes.c_int32,
                                    ctypes.c_float, ctypes.POINTER(GsGrads), ctypes.POINTER(GsGrads),
                                    ctypes.POINTER(GsAdamConfig), ctypes.c_void_p, ctypes.POINTER(GsGrads),
                                    ctypes.c_void_p]),
    "gs_train_step": (ctypes.c_int, [ctypes.POINTER(GsCamera), ctypes.c_int32, ctypes.c_int64,
                                     ctypes.POINTER(GsGrads), ctypes.c_void_p, ctypes.POINTER(GsTrainLane),
                                     ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(GsGrads),
                                     ctypes.POINTER(GsGrads), ctypes.POINTER(GsAdamConfig), ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(GsGrads), ctypes.c_void_p]),
    "gs_read_status": (ctypes.c_int, [ctypes.POINTER(GsBins), ctypes.POINTER(ctypes.c_int64),
                                      ctypes.c_void_p]),
    "gs_last_device_error": (ctypes.c_int, [ctypes.POINTER(GsBins), ctypes.c_void_p]),
    "gs_sort_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int32]),
    "gs_error_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gs_profile_begin": (ctypes.c_int, [ctypes.c_int32]),
    "gs_profile_end": (ctypes.c_int, [ctypes.POINTER(GsProfileStat), ctypes.c_int32]),
    "gs_version": (ctypes.c_int, []),
}

_LIB = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Loads libgs.so once and declares every prototype."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m gaussian_splatting_differentiable_tile_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib
