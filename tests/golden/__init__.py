"""Hand-worked expected values, each file citing the page section it follows."""
import os

HERE = os.path.dirname(os.path.abspath(__file__))


def load(name: str) -> dict:
    """Parse ``key value value ...`` lines; '#' starts a comment."""
    out = {}
    with open(os.path.join(HERE, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *vals = line.split()
            conv = []
            for v in vals:
                if v.startswith("0x"):
                    conv.append(int(v, 16))
                else:
                    try:
                        conv.append(int(v))
                    except ValueError:
                        conv.append(float(v))
            out[key] = conv if len(conv) != 1 else conv[0]
    return out
