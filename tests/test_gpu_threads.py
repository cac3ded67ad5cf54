"""Host threads sharing one device.

Each call plans its own tile width and stage count, so calls of the same
kernel can need different amounts of dynamic shared memory; the library
raises a kernel's limit once per device to the largest size any call needs,
under a lock, so calls from threads that race one another all launch.  Every
thread's results must equal a single-threaded run bit for bit (these plans
have a fixed summation order), which itself matches the FP64 oracle.
"""
import threading

import numpy as np
import pytest
import torch

import tcgen05_tmem_gemm_b200 as dg
import workloads as W
from harness import c_matrix, check_full, dg_view_of, plan, run

pytestmark = pytest.mark.gpu


def _problem(M, N, K, seed, out="f32"):
    g = torch.Generator().manual_seed(seed)
    A = W.cast(W.normal((M, K), g), "bf16")
    B = W.cast(W.normal((K, N), g), "bf16")
    return W.Problem(f"threads_{M}x{N}x{K}", W.row_major(A, "bf16"), W.row_major(B, "bf16"),
                     W.empty_out(M, N, out))


def test_threads_with_different_plans_share_a_device():
    problems = [_problem(384, 512, 320, 11), _problem(256, 64, 192, 12), _problem(1, 2048, 512, 13, "bf16")]
    plans = [plan(p.to("cuda")) for p in problems]
    # the two tensor-core plans differ in tile width or stage count, hence in shared memory
    assert plans[0]["kind_name"] == plans[1]["kind_name"] == "umma"
    assert (plans[0]["block_n"], plans[0]["stages"]) != (plans[1]["block_n"], plans[1]["stages"])
    refs = []
    for p in problems:
        check_full(p)
        refs.append(c_matrix(run(p.to("cuda"))))

    rounds = 25
    start = threading.Barrier(len(problems))
    errors = []

    def worker(k):
        try:
            gp = problems[k].to("cuda")
            s = torch.cuda.Stream()
            A, B, C = (dg_view_of(o) for o in (gp.A, gp.B, gp.C))
            start.wait(timeout=60)
            for _ in range(rounds):
                st = dg.dg_gemm(A, B, C, gp.alpha, gp.beta, None, None, s.cuda_stream)
                if st != dg.DG_OK:
                    errors.append((k, dg.status_string(st)))
                    return
            s.synchronize()
            sst = dg.dg_sync_status(s.cuda_stream)
            if sst != dg.DG_OK:
                errors.append((k, dg.status_string(sst)))
                return
            if not np.array_equal(c_matrix(gp), refs[k]):
                errors.append((k, "result differs from the single-threaded run"))
        except Exception as exc:  # reported below, in the test's thread
            errors.append((k, repr(exc)))

    threads = [threading.Thread(target=worker, args=(k,)) for k in range(len(problems))]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not any(t.is_alive() for t in threads)
    assert not errors, errors
