"""The named workloads: shapes of tensor-parallel decode all-reduce traffic.

Each workload fixes the emulated rank count, the protocols, the per-rank
message sizes, the input distribution and the chain length (operations issued
back to back in one persistent launch). Sizes are bf16 elements per rank.

* ``ll_2k``       -- 4 ranks, LL, 1024 elements (2 KB), uniform[-1,1), seed 0,
                     100 back-to-back operations on alternating parities.
* ``decode_h8192`` -- 4 ranks, sentinel, hidden 8192 x tokens {1,2,4,8}
                     (16-128 KB), normal(0,1), 160 chained operations
                     (80 layers x 2 all-reduces).
* ``decode_h4096`` -- 8 ranks, hidden 4096 x tokens {1,4,16} (8-128 KB),
                     normal(0,0.5), LL128 against the barrier oneshot and
                     twoshot baselines, 64 chained operations.
* ``sweep``       -- 1 KB .. 64 MB per rank (powers of two), 2/4/8 ranks,
                     every protocol, normal(0,1), >= 50 operations per point.
* ``allgather``   -- 8 ranks, shard 512 B .. 1 MB, uniform[-4,4), per-rank
                     start skew drawn from exponential(mean 2 us).

"SiFAR: Synchronization-Free All-Reduce for Low-Latency LLM Inference",
abstract, and "flash-comm: Self-Synchronizing Collective Communication for
LLM Decoding", abstract, motivate the decode shapes; the hidden sizes are
those of Llama-3.1-70B (8192) and Llama-3.1-8B (4096).
"""

__all__ = ["WORKLOADS", "sweep_sizes_bytes", "allgather_shard_bytes"]


def sweep_sizes_bytes():
    return [1024 << i for i in range(17)]  # 1 KB .. 64 MB


def allgather_shard_bytes():
    return [512 << i for i in range(12)]  # 512 B .. 1 MB


WORKLOADS = {
    "ll_2k": dict(nranks=4, protocols=["ll"], counts=[1024], dist="uniform",
                  params=(-1.0, 1.0), seed=0, k_ops=100),
    "decode_h8192": dict(nranks=4, protocols=["sentinel"], counts=[8192 * t for t in (1, 2, 4, 8)],
                         dist="normal", params=(1.0,), seed=0, k_ops=160),
    "decode_h4096": dict(nranks=8, protocols=["ll128", "barrier_oneshot", "barrier_twoshot"],
                         counts=[4096 * t for t in (1, 4, 16)], dist="normal", params=(0.5,),
                         seed=0, k_ops=64),
    "sweep": dict(nranks=[2, 4, 8], protocols=["ll", "ll128", "sentinel", "barrier_oneshot",
                                                "barrier_twoshot"],
                  counts=[b // 2 for b in sweep_sizes_bytes()], dist="normal", params=(1.0,),
                  seed=0, k_ops=50),
    "allgather": dict(nranks=8, protocols=["ll", "ll128", "sentinel", "barrier_oneshot"],
                      counts=[b // 2 for b in allgather_shard_bytes()], dist="uniform",
                      params=(-4.0, 4.0), seed=0, k_ops=32, skew_mean_ns=2000.0),
}
