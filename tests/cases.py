"""Parity-test workloads shared by the GPU parity tests and the CPU test that
plants mistakes in the oracle: seeded synthetic inputs that span several
tiles, ragged tails (n not a multiple of c), padding, d = 64 and 128,
c = 64, 128 and 256, bf16 and fp32."""
import workloads as wl


def _cases():
    return {
        "cfg1": lambda: wl.config_workload(1),
        "mix-fp32-d64-n1000-c64": lambda: wl.make_workload("mixture", H=2, N=1000, d=64, c=64, k=5,
                                                           dtype="fp32", seed=5),
        "lowrank-bf16-d64-n3900pad-c128": lambda: wl.make_workload("lowrank", H=3, N=4096, n_valid=3900, d=64,
                                                                   c=128, k=6, dtype="bf16", seed=6),
        "lowrank-bf16-d128-n2048-c128": lambda: wl.make_workload("lowrank", H=2, N=2048, d=128, c=128, k=4,
                                                                 dtype="bf16", seed=7),
        "mix-bf16-d64-n768-c256-tie": lambda: wl.make_workload("mixture", H=2, N=768, d=64, c=256, k=2,
                                                               dtype="bf16", seed=8),
        "single-cluster-n100-c128": lambda: wl.make_workload("mixture", H=1, N=128, n_valid=100, d=64, c=128,
                                                             k=1, dtype="bf16", seed=9),
        "n-equals-c": lambda: wl.make_workload("mixture", H=1, N=64, d=64, c=64, k=1, dtype="fp32", seed=10),
        "n-2c-plus-1": lambda: wl.make_workload("lowrank", H=2, N=320, n_valid=257, d=64, c=128, k=2,
                                                dtype="bf16", seed=11),
        "fp32-d128-n640-c64": lambda: wl.make_workload("lowrank", H=1, N=640, d=128, c=64, k=3, dtype="fp32",
                                                       seed=12),
        "grid-bf16-d128-c128": lambda: wl.make_workload("grid", H=2, N=6144, d=128, c=128, k=7, dtype="bf16",
                                                        seed=13, grid=(8, 9, 80)),
        "heavytail-bf16-d64-c256": lambda: wl.make_workload("heavytail", H=1, N=8192, d=64, c=256, k=4,
                                                            dtype="bf16", seed=14),
        # 64-key blocks on the tensor cores, with compensation blocks
        "heavytail-bf16-d64-c64": lambda: wl.make_workload("heavytail", H=1, N=8192, d=64, c=64, k=8,
                                                           dtype="bf16", seed=15),
        "lowrank-bf16-d128-c64": lambda: wl.make_workload("lowrank", H=1, N=2048, n_valid=2000, d=128, c=64,
                                                          k=5, dtype="bf16", seed=16),
    }



CASES = _cases()
