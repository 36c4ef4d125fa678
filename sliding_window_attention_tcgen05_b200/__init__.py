"""B200 (sm_100a) kernels for the Voxtral Realtime causal sliding-window encoder.

Thin PyTorch-facing binding of libvx (include/vx.h).  PyTorch provides device
memory and streams; every step of the computation runs in libvx's CUDA
kernels.  Importing this package fails when libvx.so has not been built.

Entry points (same names as the C ABI, without the ``vx_`` prefix):
  swa_attn_fwd, rms_norm_fwd, encoder_layer_fwd, conv_stem_fwd, conv_stem_step,
  encoder_fwd, log_mel_fwd, projector_fwd, stream_prefill, stream_step, pack_layer, pack_conv_weight.
"""
from ._lib import (LIB_PATH, VX_BF16, VX_F32, VxError, VxKvRing, VxLayerCfg, VxLayerWeights,  # noqa: F401
                   lib)
from .api import (ConvCache, KVRing, LayerCfg, PackedLayer, Workspace, conv_stem_fwd, conv_stem_step,  # noqa: F401
                  encoder_fwd, log_mel_fwd, projector_fwd,
                  encoder_layer_fwd, pack_conv_weight, pack_layer, rms_norm_fwd, selftest_wait_timeout,
                  set_wait_timeout_ns, status_check, status_reset, stream_prefill, stream_step,
                  swa_attn_fwd, VOXTRAL_RT)

__version__ = lib.vx_version().decode()
