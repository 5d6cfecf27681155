"""Python binding of the KLA C ABI (filled in with the CUDA library)."""


class KLAError(RuntimeError):
    pass


def chunk_fwd(*a, **k):
    raise KLAError("CUDA library not built yet")


def decode_step(*a, **k):
    raise KLAError("CUDA library not built yet")


def chunk_fwd_workspace_size(*a, **k):
    raise KLAError("CUDA library not built yet")
