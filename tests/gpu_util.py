"""Helpers for the GPU tests: move generator/oracle numpy arrays to and from
the device (bit patterns are preserved exactly)."""
import numpy as np
import torch

DEV = "cuda"


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(DEV)


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(DEV)


def dev_i32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(DEV)


def host_bits16(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def u32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def rel_frob(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def oracle_rows(fn, rows, chunk: int = 4):
    """Run fn(list_of_rows) -> array over `rows` in chunks on a thread pool and
    concatenate in row order.  The oracle is C called through ctypes, which
    releases the GIL, so the chunks run on all host cores without copying the
    (large) shared inputs."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    rows = list(rows)
    parts = [rows[i:i + chunk] for i in range(0, len(rows), chunk)]
    with ThreadPoolExecutor(max_workers=max(1, min(len(parts), os.cpu_count() or 1))) as ex:
        outs = list(ex.map(fn, parts))
    return np.concatenate(outs, axis=0)


def sample_rows(seed: int, n_total: int, count: int, must=()):
    """`count` distinct row indices of [0, n_total): the `must` rows first, then
    seeded uniform picks (SplitMix64 through the input generator)."""
    import synth
    rows = list(dict.fromkeys(int(r) for r in must))
    cand = synth.permutation(seed, n_total)
    for r in cand:
        if len(rows) >= count:
            break
        if int(r) not in rows:
            rows.append(int(r))
    return np.array(sorted(rows), dtype=np.int64)
