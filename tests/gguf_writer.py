"""A minimal GGUF writer for the reader's tests (test infrastructure).

Writes the public GGUF layout, version 3, little-endian: "GGUF", u32
version, u64 tensor count, u64 metadata count; metadata as (string key, u32
type, value); tensor infos as (string name, u32 n_dims, u64 dims[n_dims]
innermost first, u32 ggml type, u64 offset from the data section); then
padding to the alignment and the tensor bytes, each at a multiple of it.
A string is u64 length + bytes; an array is u32 element type + u64 count +
elements.
"""
import struct

# GGUF metadata value types
U8, I8, U16, I16, U32, I32, F32, BOOL, STRING, ARRAY, U64, I64, F64 = range(13)
_FMT = {U8: "<B", I8: "<b", U16: "<H", I16: "<h", U32: "<I", I32: "<i", F32: "<f", BOOL: "<?", U64: "<Q",
        I64: "<q", F64: "<d"}


def _str(s: str) -> bytes:
    b = s.encode()
    return struct.pack("<Q", len(b)) + b


def _value(t: int, v) -> bytes:
    if t == STRING:
        return _str(v)
    if t == ARRAY:
        et, items = v
        return struct.pack("<IQ", et, len(items)) + b"".join(_value(et, x) for x in items)
    return struct.pack(_FMT[t], v)


def write(path, tensors, metadata=(), alignment=32, version=3, magic=b"GGUF", offsets=None, truncate=0):
    """tensors: list of (name, ggml_type, dims (innermost first), bytes).
    metadata: list of (key, type, value).  offsets: explicit data offsets
    (else each tensor at the next multiple of `alignment`).  truncate: bytes
    cut from the end of the file."""
    meta = list(metadata)
    if alignment != 32:
        meta.append(("general.alignment", U32, alignment))
    head = magic + struct.pack("<IQQ", version, len(tensors), len(meta))
    for k, t, v in meta:
        head += _str(k) + struct.pack("<I", t) + _value(t, v)
    offs, off = [], 0
    for _, _, _, data in tensors:
        off = (off + alignment - 1) // alignment * alignment
        offs.append(off)
        off += len(data)
    if offsets is not None:
        offs = list(offsets)
    for (name, gt, dims, _), o in zip(tensors, offs):
        head += _str(name) + struct.pack("<I", len(dims)) + b"".join(struct.pack("<Q", d) for d in dims)
        head += struct.pack("<IQ", gt, o)
    start = (len(head) + alignment - 1) // alignment * alignment
    out = bytearray(head + b"\0" * (start - len(head)))
    for (_, _, _, data), o in zip(tensors, offs):
        end = start + o
        if len(out) < end:
            out += b"\0" * (end - len(out))
        out[end:end + len(data)] = bytes(data)
    if truncate:
        out = out[:-truncate]
    with open(path, "wb") as f:
        f.write(out)
