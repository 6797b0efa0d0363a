"""libmla: MLA latent-KV decode for B200 (sm_100a).

* :mod:`.binding`   — ctypes binding of the C ABI in ``include/mla.h``
  (``mla_decode_plan`` / ``mla_decode`` / ``mla_combine`` / ...).
* :mod:`.decoder`   — ``MlaDecoder``: buffers plus the three calls on a stream.
* :mod:`.workloads` — seeded synthetic inputs.
* :mod:`.build`     — builds ``libmla.so`` in-tree with nvcc.

The binding loads lazily, so that input generation and the build work
without the library; touching any binding name without ``libmla.so`` raises.
"""

_BINDING_NAMES = {
    "mla_plan_bytes", "mla_workspace_bytes", "mla_num_workers", "mla_decode_plan", "mla_decode", "mla_combine",
    "mla_get_error", "mla_status_string", "mla_decode_desc_t", "make_desc", "MlaError",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding

        return getattr(binding, name)
    if name in ("MlaDecoder", "decoder_for"):
        from . import decoder

        return getattr(decoder, name)
    raise AttributeError(name)
