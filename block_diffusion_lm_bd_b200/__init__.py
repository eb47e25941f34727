"""B200-native denoise step of a block-diffusion language model.

One denoising step of an active block of S masked tokens:

* ``attn_step`` - the block queries attend to a cached clean-prefix KV and,
  bidirectionally, to the block's own KV, merged in one online softmax
  (split-KV over the prefix, log-sum-exp combine across splits);
* ``unmask`` - full-vocabulary softmax per masked position, argmax token and
  its probability (confidence), commit where confidence > gamma.

Every step runs in the CUDA kernels of ``libbd.so`` (sm_100a), reached through
its C ABI (``include/bd.h``). This package only marshals arguments; there is
no CPU fallback. Importing the package loads nothing; the first call into
``api`` loads the library and raises if it is missing.
"""

_API = (
    "BdError",
    "attn_step",
    "attn_workspace_bytes",
    "unmask",
    "unmask_workspace_bytes",
    "get_device_status",
    "status_string",
    "lib_path",
)


def __getattr__(name):
    if name in _API:
        from . import api

        return getattr(api, name)
    raise AttributeError(name)


__all__ = list(_API)
