"""placeholder"""
FA_OK = 0
FA_ERR_INVALID_ARG = 1
FA_ERR_UNSUPPORTED = 2
FA_ERR_MISALIGNED = 3
FA_ERR_CUDA = 4
FA_ERR_TIMEOUT = 5
class FaError(RuntimeError):
    pass
library = library_path = fa_fwd = fa_bwd = fa_bwd_workspace_size = None
fa_get_device_error = fa_strerror = attention_forward = attention_backward = None
