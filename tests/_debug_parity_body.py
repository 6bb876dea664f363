"""Run by tests/test_gpu_debug_build.py in a subprocess whose SFC_LIB points
at libsfc_debug.so (every scratch access bounds-checked on the device). Every
protocol, several rank counts, ragged sizes; outputs bit-exact to the oracle,
status OK (an out-of-region access would have recorded SFC_ERR_GUARD), guard
words intact. Exit code 0 on success."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from _gpu_helpers import run_chain  # noqa: E402

from latency_self_synchronizing_b200 import _lib, api  # noqa: E402
from latency_self_synchronizing_b200.inputs import make_inputs  # noqa: E402
from oracle import reference  # noqa: E402

AR = ["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_twoshot", "barrier_oneshot_db", "ll_twoshot",
      "sentinel_twoshot", "ll128_fast"]
AG = ["ll", "ll128", "sentinel", "barrier_oneshot", "barrier_oneshot_db", "ll128_fast"]


def main():
    assert _lib.LIB_PATH.endswith("libsfc_debug.so"), _lib.LIB_PATH
    cases = 0
    for n in (2, 3, 5, 8):
        comm = api.Communicator(n, 1 << 14)
        try:
            for count in (1, 61, 1000, 4099):
                for proto in AR:
                    x = make_inputs(seed=count * 10 + n, k_ops=3, nranks=n, count=count)
                    out = run_chain(comm, proto, x)
                    for k in range(3):
                        for r in range(n):
                            np.testing.assert_array_equal(out[k, r], reference.allreduce(x[k]))
                    cases += 1
                for proto in AG:
                    c = max(1, count // n)
                    x = make_inputs(seed=count * 10 + n + 1, k_ops=2, nranks=n, count=c)
                    out = run_chain(comm, proto, x, op="allgather")
                    for k in range(2):
                        for r in range(n):
                            np.testing.assert_array_equal(out[k, r], reference.allgather(x[k]))
                    cases += 1
            assert comm.check_guards() == api.Status.OK
        finally:
            comm.close()
    # the allocation-free entry point on its static scratch
    import torch
    x = make_inputs(seed=99, k_ops=1, nranks=4, count=1000)
    ins = [torch.from_numpy(x[0, r].view(np.int16)).cuda().view(torch.bfloat16) for r in range(4)]
    outs = [torch.empty_like(t) for t in ins]
    import ctypes as C
    lib = _lib.load()
    pin = (C.c_void_p * 4)(*[t.data_ptr() for t in ins])
    pout = (C.c_void_p * 4)(*[t.data_ptr() for t in outs])
    assert lib.sfc_allreduce_noalloc(pin, pout, 4, 1000, C.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    torch.cuda.synchronize()
    for r in range(4):
        np.testing.assert_array_equal(outs[r].view(torch.int16).cpu().numpy().view(np.uint16),
                                      reference.allreduce(x[0]))
    cases += 1
    print(f"debug build: {cases} chains bit-exact, no out-of-region scratch access")


if __name__ == "__main__":
    main()
