"""wav2vec2-style CTC forward pass on B200: a C-ABI CUDA library (libw2v.so,
built from csrc/ for sm_100a) and its thin Python binding."""
from .w2v import (Model, W2VError, lib, make_config, w2v_config, w2v_create, w2v_ctc_greedy, w2v_debug_read,
                  w2v_destroy, w2v_forward, w2v_num_frames, w2v_sync, w2v_weight_count, w2v_weight_manifest)

__all__ = ["Model", "W2VError", "lib", "make_config", "w2v_config", "w2v_create", "w2v_ctc_greedy",
           "w2v_debug_read", "w2v_destroy", "w2v_forward", "w2v_num_frames", "w2v_sync", "w2v_weight_count",
           "w2v_weight_manifest"]
