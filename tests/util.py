"""Helpers shared by the tests: host <-> device copies of rank buffers and
bit-level comparison.  No collective arithmetic lives here."""
import numpy as np

NP = {"f32": np.float32, "bf16": np.uint16, "i32": np.int32}


def to_dev(xs, dt, device="cuda", pad_bytes=0, offset_bytes=0):
    """Copy host rank buffers to the device.  offset_bytes shifts each buffer
    inside a slightly larger allocation (misaligned starts); pad_bytes adds a
    canary region after each buffer.  Returns (tensors, backing)."""
    import torch
    out, backing = [], []
    for x in xs:
        raw = np.ascontiguousarray(x).view(np.uint8)
        total = offset_bytes + raw.size + pad_bytes
        buf = torch.empty(total + 16, dtype=torch.uint8, device=device)
        buf.fill_(0xA5)
        base = offset_bytes
        buf[base:base + raw.size].copy_(torch.from_numpy(raw))
        backing.append(buf)
        out.append(_typed(buf[base:base + raw.size], dt))
    torch.cuda.synchronize()
    return out, backing


def empty_dev(n, dt, count, device="cuda", pad_bytes=64, offset_bytes=0, fill=0x5A):
    """count device buffers of n elements, each followed by a canary band."""
    import torch
    esz = np.dtype(NP[dt]).itemsize
    outs, backing = [], []
    for _ in range(count):
        buf = torch.full((offset_bytes + n * esz + pad_bytes + 16,), fill, dtype=torch.uint8,
                         device=device)
        backing.append(buf)
        outs.append(_typed(buf[offset_bytes:offset_bytes + n * esz], dt))
    torch.cuda.synchronize()
    return outs, backing


def _typed(u8, dt):
    import torch
    if u8.numel() == 0:
        return u8.view(torch.int16).view(torch.bfloat16) if dt == "bf16" else \
            u8.view(torch.float32 if dt == "f32" else torch.int32)
    if dt == "f32":
        return u8.view(torch.float32)
    if dt == "bf16":
        return u8.view(torch.int16).view(torch.bfloat16)
    return u8.view(torch.int32)


def to_host(t, dt):
    import torch
    if dt == "bf16":
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy().astype(NP[dt], copy=False)


def bits(a):
    a = np.asarray(a)
    if a.dtype == np.float32:
        return a.view(np.uint32)
    return a


def assert_bits(got, want, what=""):
    g, w = bits(got), bits(want)
    if g.shape != w.shape or not np.array_equal(g, w):
        bad = np.nonzero(g != w)[0] if g.shape == w.shape else []
        i = int(bad[0]) if len(bad) else -1
        raise AssertionError(f"{what}: {len(bad)} mismatching elements; first at {i}: "
                             f"got {g[i] if i >= 0 else g.shape} want {w[i] if i >= 0 else w.shape}")


def check_canary(backing, start_bytes, fill=0x5A, what="canary"):
    """Bytes from start_bytes to the end of each backing buffer must still hold fill."""
    for k, b in enumerate(backing):
        tail = b[start_bytes:].cpu().numpy()
        if not np.all(tail == fill):
            raise AssertionError(f"{what}[{k}]: out-of-bounds write past the output")
