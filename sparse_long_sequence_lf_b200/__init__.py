"""Longformer self-attention on B200 (sm_100a): forward, backward, and the
projection and output layers around it.

The compute path is the CUDA library under ``csrc/`` behind the C ABI
``include/lf_attention.h``; ``api`` is its thin Python binding.  Importing this
package loads nothing; the first API call loads the library and raises if it
is missing.
"""
from .api import (attention_backward, attention_forward, attention_forward_host,
                  attention_forward_static, attention_prepare, attention_run,
                  backward_scratch_size, encoder_forward, encoder_workspace_size, ffn_block,
                  ffn_workspace_size, global_index, host_copy_bytes, host_staging_size,
                  new_workspace, output_layer, output_workspace_size, qkv_projection, scratch_status,
                  workspace_size, workspace_status)
from ._lib import LfError

__all__ = ["attention_backward", "attention_forward", "attention_forward_host",
           "attention_forward_static", "attention_prepare", "attention_run",
           "backward_scratch_size", "encoder_forward", "encoder_workspace_size", "ffn_block",
           "ffn_workspace_size", "global_index", "host_copy_bytes", "host_staging_size",
           "new_workspace",
           "output_layer", "output_workspace_size", "qkv_projection", "scratch_status",
           "workspace_size", "workspace_status", "LfError"]
