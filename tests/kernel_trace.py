"""Names of the GPU kernels a call launches, read from the torch profiler
(a test helper).  The profiler's kernel records occasionally come back empty
while the runtime records are present; the call is then profiled again."""
import torch
from torch.autograd import DeviceType


def kernel_names(fn, tries: int = 3) -> list:
    from torch.profiler import ProfilerActivity, profile
    for _ in range(tries):
        fn()
        torch.cuda.synchronize()
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type == DeviceType.CUDA]
        if names:
            return names
    return []
